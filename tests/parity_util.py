"""Comparison rules between the CUDA path and the fp64 oracle.

Scores: |s_gpu - s_ref| <= 1e-3 |s_ref| + 1e-30 at every position.
Index sets: with T the oracle's k_sel-th largest pooled candidate score, every candidate
with s~_ref > T (1 + 1e-3) must be kept and every one with s~_ref < T (1 - 1e-3) must not;
only candidates inside that band may differ.  The count, the sinks, the window and the
ascending order are exact.  Gathered rows are bit-exact given the GPU's own indices.
"""
import numpy as np
import torch

SCORE_RTOL = 1e-3


def check_scores(gpu, ref, rtol=SCORE_RTOL):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = rtol * np.abs(ref) + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{bad.sum()} scores outside tolerance; worst rel "
                           f"{(err / np.maximum(np.abs(ref), 1e-30)).max():.3e}")
    return float((err / np.maximum(np.abs(ref), 1e-30)).max())


def check_index_row(idx, pooled_ref, N, S, w, budget, rtol=SCORE_RTOL):
    """Band rule for one row; returns True if the set equals the oracle's exactly."""
    idx = np.asarray(idx)
    assert idx.shape == (budget,)
    assert np.all(np.diff(idx) > 0), "kept positions not strictly ascending"
    assert idx[0] >= 0 and idx[-1] < N
    kept = set(idx.tolist())
    assert set(range(S)) <= kept, "sinks not kept"
    assert set(range(N - w, N)) <= kept, "recent window not kept"
    sel = np.array(sorted(kept - set(range(S)) - set(range(N - w, N))), dtype=np.int64)
    k_sel = budget - S - w
    assert sel.size == k_sel
    cand = pooled_ref[S:N - w]
    order = sorted(range(cand.size), key=lambda i: (-cand[i], i))
    T = cand[order[k_sel - 1]]
    must = S + np.nonzero(cand > T * (1 + rtol))[0]
    mustnot = S + np.nonzero(cand < T * (1 - rtol))[0]
    missing = np.setdiff1d(must, sel)
    extra = np.intersect1d(mustnot, sel)
    assert missing.size == 0, f"{missing.size} clearly-above-threshold tokens dropped"
    assert extra.size == 0, f"{extra.size} clearly-below-threshold tokens kept"
    ref_sel = np.sort(S + np.array(order[:k_sel]))
    return bool(np.array_equal(ref_sel, sel))


def check_index_sets(idx, pooled_ref, N, S, w, budget):
    idx = np.asarray(idx)
    rows = idx.reshape(-1, budget)
    ref = pooled_ref.reshape(-1, N)
    exact = [check_index_row(rows[r], ref[r], N, S, w, budget) for r in range(rows.shape[0])]
    return sum(exact) / len(exact)


def check_gather(out, src, idx):
    """out [B, H, K, ...] must equal src[b, h, idx[b, h' , :]] bit for bit."""
    B, H = out.shape[:2]
    Hidx = idx.shape[1]
    src_i = src.view(torch.int16) if src.dtype == torch.bfloat16 else src.view(torch.int32)
    out_i = out.view(torch.int16) if out.dtype == torch.bfloat16 else out.view(torch.int32)
    idx_t = torch.as_tensor(np.asarray(idx), device=src.device).long()
    for b in range(B):
        for h in range(H):
            want = src_i[b, h].index_select(0, idx_t[b, 0 if Hidx == 1 else h])
            assert torch.equal(out_i[b, h], want), f"gathered rows differ at b={b} h={h}"
