"""Decode-time KV cache kept within a budget by CentroidKV's periodic clustering.

CentroidKV page, sec. 2 "Inferentie Pipeline": after prefill a first clustering round runs
when the cache exceeds the budget; during decoding the cache grows by one token per step
and a round runs every g steps; sinks and recent tokens are preserved.  Sec. 3 "Progressive
Scheduling": round j merges with ratio r_j = r_init - j * delta.  Sec. 4: attention runs
over the centroids with ln(degree) added to the logits.

This class only holds the buffers and the schedule; every step runs in the library's
kernels (kvc_append, kvc_csm, kvc_decode_attention).  Two buffer sets of capacity `cap`
alternate as the input and the output of a round.  Order inside a decode step: the new
tokens are appended, the queries attend to the cache (new tokens included), and every g-th
step then runs a round if the cache holds more than `budget` tokens.
"""
from __future__ import annotations

import torch

from . import kvc


class CentroidCache:
    def __init__(self, B: int, H: int, capacity: int, *, budget: int, n_sink: int, window: int, chunk: int,
                 r_init: float, delta: float, g: int, dtype=torch.bfloat16, device="cuda", D: int = 128):
        if capacity < 1 or budget < 1 or g < 1:
            raise ValueError("capacity, budget and g must be positive")
        if not (0.0 <= r_init <= 0.5) or delta < 0.0:
            raise ValueError("the merge ratio starts in [0, 0.5] and does not grow")
        self.B, self.H, self.cap, self.D = B, H, capacity, D
        self.budget, self.n_sink, self.window, self.chunk = budget, n_sink, window, chunk
        self.r_init, self.delta, self.g = r_init, delta, g
        self.k = [torch.empty((B, H, capacity, D), dtype=dtype, device=device) for _ in range(2)]
        self.v = [torch.empty((B, H, capacity, D), dtype=dtype, device=device) for _ in range(2)]
        self.deg = [torch.empty((B, H, capacity), dtype=torch.int32, device=device) for _ in range(2)]
        self.pos = [torch.empty((B, H, capacity), dtype=torch.int32, device=device) for _ in range(2)]
        self.cur = 0          # buffer set holding the cache
        self.n = 0            # tokens (centroids) in the cache, the same for every (b, h)
        self.seen = 0         # tokens appended so far (the next position)
        self.round = 0        # clustering rounds run so far
        self.steps = 0        # decode steps taken
        self._ws = None

    # views of the live cache
    def view(self):
        c = self.cur
        return {"k": self.k[c][:, :, :self.n], "v": self.v[c][:, :, :self.n], "deg": self.deg[c][:, :, :self.n],
                "pos": self.pos[c][:, :, :self.n]}

    def _append(self, k_new, v_new):
        t = k_new.shape[2]
        if self.n + t > self.cap:
            raise RuntimeError(f"cache capacity {self.cap} exceeded ({self.n} + {t})")
        c = self.cur
        kvc.kvc_append(self.k[c], self.v[c], self.n, k_new.contiguous(), v_new.contiguous(), deg_cache=self.deg[c],
                       pos_cache=self.pos[c], pos0=self.seen)
        self.n += t
        self.seen += t

    def compress(self) -> int:
        """One clustering round with this round's ratio; returns the number of merges."""
        r = kvc.kvc_csm_ratio(self.r_init, self.delta, self.round)
        self.round += 1
        m = kvc.kvc_csm_merges(self.n, self.n_sink, self.window, self.chunk, r)
        if m <= 0:
            return 0
        c, o = self.cur, 1 - self.cur
        kvc.kvc_csm(self.k[c], self.v[c], self.n_sink, self.window, self.chunk, r, deg=self.deg[c], n=self.n,
                    pos=self.pos[c], out={"k_out": self.k[o], "v_out": self.v[o], "deg_out": self.deg[o],
                                          "pos_out": self.pos[o]}, ws=self._round_ws(r))
        self.cur = o
        self.n -= m
        return m

    def _round_ws(self, r):
        need = kvc.kvc_csm_workspace_size(self.B, self.H, self.n, self.n_sink, self.window, self.chunk, r)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.k[0].device)
        return self._ws

    def prefill(self, k, v) -> int:
        """Loads the prompt's K and V [B, H, N, D]; runs the first round if over budget."""
        self._append(k, v)
        return self.compress() if self.n > self.budget else 0

    def step(self, q, k_new, v_new):
        """One decode step: append k_new, v_new [B, H, t, D], attend with q [B, Hq, nq, D]
        over the cache, then cluster if this is a g-th step and the cache is over budget.
        Returns the attention output [B, Hq, nq, D] fp32."""
        self._append(k_new, v_new)
        c = self.cur
        out = kvc.kvc_decode_attention(q, self.k[c], self.v[c], deg=self.deg[c], n=self.n)
        self.steps += 1
        if self.steps % self.g == 0 and self.n > self.budget:
            self.compress()
        return out
