"""Writes oracle_regression.json: outputs of the fp64 oracle on tiny closed-form inputs.

The pages print no worked numerical example, so nothing here is a page value and nothing
here pins the oracle's correctness (tests/test_oracle_pins.py does that against closed
forms, library routines and brute force).  These values guard the oracle against silent
change: tests/test_golden.py recomputes them, and a change to the oracle's arithmetic must
regenerate this file with the passage that justifies it named in the commit message.

Inputs are closed-form (no random generator): element i of a tensor with salt c is
sin(0.37 i + 0.11 c) + 0.25 cos(0.053 i * i + c).  Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import math
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
from oracle import oracle as O  # noqa: E402


def closed_form(shape, salt):
    n = int(np.prod(shape))
    i = np.arange(n, dtype=np.float64)
    x = np.sin(0.37 * i + 0.11 * salt) + 0.25 * np.cos(0.053 * i * i + salt)
    return torch.from_numpy(x.reshape(shape))


def cases():
    out = {}
    # score -> pool -> select: B1, Hq 4 / Hkv 2, N 40, w 4, D 16, S 1, pool 3, budget 12
    q = closed_form((1, 4, 4, 16), 1)
    k = closed_form((1, 2, 40, 16), 2)
    s = O.score(q, k, window=4)
    pooled = O.pool(s, 1, 36, 3)
    idx = O.select(pooled, 1, 4, 12)
    out["saliency"] = {"shapes": {"q": [1, 4, 4, 16], "k": [1, 2, 40, 16]}, "salts": {"q": 1, "k": 2},
                       "window": 4, "n_sink": 1, "pool_kernel": 3, "budget": 12,
                       "scores": s.tolist(), "pooled": pooled[:, :, 1:36].tolist(), "idx": idx.tolist()}
    # one Chunked Soft Matching round: one row of 30 tokens, D 16, S 1, w 3, chunk 6, r 0.4
    kc = closed_form((1, 30, 16), 3)
    vc = closed_form((1, 30, 16), 4)
    deg = (np.arange(30) % 3 + 1).astype(np.int32).reshape(1, 30)
    r = O.csm(kc, vc, deg, n_sink=1, window=3, chunk=6, ratio=0.4)
    out["csm"] = {"shapes": {"k": [1, 30, 16], "v": [1, 30, 16]}, "salts": {"k": 3, "v": 4},
                  "deg": "i % 3 + 1", "n_sink": 1, "window": 3, "chunk": 6, "ratio": 0.4,
                  "m": r["m"], "pos_out": r["pos_out"].tolist(), "deg_out": r["deg_out"].tolist(),
                  "k_out": r["k_out"].tolist(), "v_out": r["v_out"].tolist()}
    # decode attention over centroids: q [1, 4, 2, 16], cache [1, 2, 9, 16], degrees i % 4 + 1
    qd = closed_form((1, 4, 2, 16), 5)
    kd = closed_form((1, 2, 9, 16), 6)
    vd = closed_form((1, 2, 9, 16), 7)
    dd = (np.arange(18) % 4 + 1).astype(np.int32).reshape(1, 2, 9)
    att = O.centroid_attention(qd, kd, vd, dd)
    out["decode_attention"] = {"shapes": {"q": [1, 4, 2, 16], "k": [1, 2, 9, 16], "v": [1, 2, 9, 16]},
                               "salts": {"q": 5, "k": 6, "v": 7}, "deg": "i % 4 + 1", "out": att.tolist()}
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        json.dump(cases(), f, indent=1)
        f.write("\n")
    print("wrote", os.path.join(HERE, "oracle_regression.json"))
