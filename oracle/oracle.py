"""Python front of the fp64 CPU oracle (kvc_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's CPU-baseline
leg may import this module; the product path never does.  It imports nothing from the
CUDA library package.

All arithmetic lives in kvc_oracle.c (fp64, plain loops).  This file only marshals
arguments and composes the steps in the order the method takes them:
score -> aggregate -> pool -> select -> gather (+ the TSP branch), plus the pivot metrics
(attention entropy of the window rows, kept mass and candidate variance of score rows),
CentroidKV's Chunked Soft Matching round and decode attention over its centroids.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvc_oracle.c")
_SO = os.path.join(_HERE, "libkvc_oracle.so")

F32, BF16, F64 = 0, 1, 2
SCOPE_PER_KV_HEAD, SCOPE_ALL_HEADS = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile kvc_oracle.c into libkvc_oracle.so (plain -O2, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-o", _SO, _SRC, "-lm", "-lpthread"])
    return _SO


def _load(so_path: str):
    L = ctypes.CDLL(so_path)
    i, p, d, sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_double, ctypes.c_size_t
    L.oracle_score.argtypes = [i, i, i, i, i, i, i, i, p, p, i, p, i]
    L.oracle_accumulate.argtypes = [p, p, i, i, i, i]
    L.oracle_pool.argtypes = [p, p, i, i, i, i, i, i]
    L.oracle_select.argtypes = [p, i, i, i, i, i, i, p]
    L.oracle_gather.argtypes = [p, i, i, i, sz, p, i, i, p]
    L.oracle_tsp_count.argtypes = [i, i, i, d]
    L.oracle_entropy.argtypes = [i, i, i, i, i, i, i, p, p, i, p, i, p, i]
    L.oracle_row_stats.argtypes = [p, i, i, i, i, p, i, p, p]
    L.oracle_csm_merges.argtypes = [i, i, i, i, d]
    L.oracle_csm.argtypes = [p, p, i, p, i, i, i, i, i, i, d, p, p, p, p, p, p, p]
    L.oracle_csm_ratio.argtypes = [d, d, i]
    L.oracle_centroid_attention.argtypes = [p, i, p, p, i, p, i, i, i, i, i, i, p]
    L.oracle_csm_ratio.restype = d
    for f in ("oracle_score", "oracle_accumulate", "oracle_pool", "oracle_select",
              "oracle_gather", "oracle_tsp_count", "oracle_entropy", "oracle_row_stats",
              "oracle_csm_merges", "oracle_csm", "oracle_centroid_attention"):
        getattr(L, f).restype = ctypes.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _load(_SO)
    return _lib


class using_library:
    """Temporarily route every oracle call to another build of kvc_oracle.c (used by the
    test that checks the pins reject deliberately broken copies of the oracle)."""

    def __init__(self, so_path: str):
        self.so_path = so_path

    def __enter__(self):
        global _lib
        self.saved = lib()
        _lib = _load(self.so_path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _as_buffer(x):
    """A C-contiguous CPU numpy view/copy of x and its oracle dtype code."""
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy(), BF16
        if x.dtype == torch.float32:
            return x.numpy(), F32
        if x.dtype == torch.float64:
            return x.numpy(), F64
        raise TypeError(f"unsupported dtype {x.dtype}")
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.float64:
        return x, F64
    raise TypeError(f"unsupported dtype {x.dtype}")


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments")


def score(q, k, *, window: int, scope: int = SCOPE_PER_KV_HEAD, threads: int = 0) -> np.ndarray:
    """Saliency scores in fp64.

    q [L, B, Hq, w, D] (or [B, Hq, w, D] for one layer), k [L, B, Hkv, N, D] (or [B, Hkv, N, D]).
    Returns [B, Hkv, N] (scope PER_KV_HEAD) or [B, 1, N] (scope ALL_HEADS), summed over layers.
    """
    if q.dim() == 4:
        q, k = q.unsqueeze(0), k.unsqueeze(0)
    L, B, Hq, w, D = q.shape
    _, _, Hkv, N, _ = k.shape
    assert w == window and k.shape[0] == L and k.shape[1] == B and k.shape[4] == D
    qb, qd = _as_buffer(q)
    kb, kd = _as_buffer(k)
    assert qd == kd
    Hs = Hkv if scope == SCOPE_PER_KV_HEAD else 1
    out = np.zeros((B, Hs, N), dtype=np.float64)
    threads = threads or (os.cpu_count() or 1)
    rc = lib().oracle_score(B, Hq, Hkv, N, D, w, L, scope, qb.ctypes.data, kb.ctypes.data, qd,
                            out.ctypes.data, threads)
    _check(rc, "score")
    return out


def accumulate(acc: np.ndarray, src: np.ndarray) -> np.ndarray:
    """acc[B, Ho, N] += group sums of src[B, Hi, N] (Hi % Ho == 0); returns acc."""
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    src = np.ascontiguousarray(src, dtype=np.float64)
    B, Ho, N = acc.shape
    Hi = src.shape[1]
    _check(lib().oracle_accumulate(acc.ctypes.data, src.ctypes.data, B, Hi, Ho, N), "accumulate")
    return acc


def pool(x: np.ndarray, lo: int, hi: int, kernel: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    B, H, N = x.shape
    out = np.empty_like(x)
    _check(lib().oracle_pool(x.ctypes.data, out.ctypes.data, B, H, N, lo, hi, kernel), "pool")
    return out


def select(pooled: np.ndarray, n_sink: int, window: int, budget: int) -> np.ndarray:
    pooled = np.ascontiguousarray(pooled, dtype=np.float64)
    B, H, N = pooled.shape
    idx = np.empty((B, H, budget), dtype=np.int32)
    _check(lib().oracle_select(pooled.ctypes.data, B, H, N, n_sink, window, budget, idx.ctypes.data),
           "select")
    return idx


def gather(src: torch.Tensor, idx: np.ndarray) -> torch.Tensor:
    """src [B, Hsrc, N, row...] (any dtype), idx [B, Hidx, K] -> [B, Hsrc, K, row...]."""
    src = src.detach().cpu().contiguous()
    B, Hsrc, N = src.shape[:3]
    row_bytes = src[0, 0, 0].numel() * src.element_size()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    Hidx, K = idx.shape[1], idx.shape[2]
    dst = torch.empty((B, Hsrc, K) + tuple(src.shape[3:]), dtype=src.dtype)
    sb = src.view(torch.uint8).numpy() if src.dtype != torch.uint8 else src.numpy()
    db = dst.view(torch.uint8).numpy() if dst.dtype != torch.uint8 else dst.numpy()
    _check(lib().oracle_gather(sb.ctypes.data, B, Hsrc, N, row_bytes, idx.ctypes.data, Hidx, K,
                               db.ctypes.data), "gather")
    return dst


def tsp_count(N: int, window: int, n_sink: int, rate: float) -> int:
    return int(lib().oracle_tsp_count(N, window, n_sink, float(rate)))


def entropy(q, k, *, window: int, rows=None, threads: int = 0) -> np.ndarray:
    """Attention entropy (nats) of window query rows, fp64.

    q [L, B, Hq, w, D] (or [B, Hq, w, D]), k [L, B, Hkv, N, D] (or [B, Hkv, N, D]).  Returns
    [L, B, Hq, w], or, with `rows` (flat indices into that shape), the listed rows only.
    """
    if q.dim() == 4:
        q, k = q.unsqueeze(0), k.unsqueeze(0)
    L, B, Hq, w, D = q.shape
    _, _, Hkv, N, _ = k.shape
    assert w == window and k.shape[0] == L and k.shape[1] == B and k.shape[4] == D
    qb, qd = _as_buffer(q)
    kb, kd = _as_buffer(k)
    assert qd == kd
    all_rows = rows is None
    r = np.arange(L * B * Hq * w, dtype=np.int32) if all_rows else np.ascontiguousarray(rows, dtype=np.int32)
    out = np.zeros(r.size, dtype=np.float64)
    threads = threads or (os.cpu_count() or 1)
    rc = lib().oracle_entropy(B, Hq, Hkv, N, D, w, L, qb.ctypes.data, kb.ctypes.data, qd, r.ctypes.data, r.size,
                              out.ctypes.data, threads)
    _check(rc, "entropy")
    return out.reshape(L, B, Hq, w) if all_rows else out


def row_stats(scores: np.ndarray, n_sink: int, window: int, idx: np.ndarray = None):
    """(kept_mass, cand_var) per score row of scores [B, H, N] (kept_mass None without idx)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    B, H, N = s.shape
    km = np.zeros((B, H), dtype=np.float64)
    cv = np.zeros((B, H), dtype=np.float64)
    ip, budget = None, 0
    if idx is not None:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        budget = idx.shape[-1]
        ip = idx.ctypes.data
    rc = lib().oracle_row_stats(s.ctypes.data, B * H, N, n_sink, window, ip, budget, km.ctypes.data,
                                cv.ctypes.data)
    _check(rc, "row_stats")
    return (km if idx is not None else None), cv


def csm_merges(N: int, n_sink: int, window: int, chunk: int, ratio: float) -> int:
    m = int(lib().oracle_csm_merges(N, n_sink, window, chunk, float(ratio)))
    _check(0 if m >= 0 else -1, "csm_merges")
    return m


def csm_ratio(r_init: float, delta: float, round_: int) -> float:
    return float(lib().oracle_csm_ratio(float(r_init), float(delta), int(round_)))


def csm(k, v, deg, *, n_sink: int, window: int, chunk: int, ratio: float) -> dict:
    """One Chunked Soft Matching round (fp64) over k, v [..., N, D] (fp32 / bf16 / fp64 tensors)
    with degrees deg [..., N] int32.  Returns best, sim, merged [..., N] and the kept
    k_out, v_out [..., N - m, D] (input dtype), deg_out, pos_out [..., N - m]."""
    k = k.detach().cpu().contiguous()
    v = v.detach().cpu().contiguous()
    lead, (N, D) = tuple(k.shape[:-2]), tuple(k.shape[-2:])
    rows = int(np.prod(lead)) if lead else 1
    kb, kd = _as_buffer(k)
    vb, vd = _as_buffer(v)
    assert kd == vd and v.shape == k.shape
    dg = np.ascontiguousarray(np.asarray(deg, dtype=np.int32).reshape(rows, N))
    m = csm_merges(N, n_sink, window, chunk, ratio)
    n_out = N - m
    best = np.empty((rows, N), dtype=np.int32)
    sim = np.empty((rows, N), dtype=np.float64)
    merged = np.empty((rows, N), dtype=np.uint8)
    k_out = torch.empty(lead + (n_out, D), dtype=k.dtype)
    v_out = torch.empty(lead + (n_out, D), dtype=k.dtype)
    ko, _ = _as_buffer(k_out)
    vo, _ = _as_buffer(v_out)
    deg_out = np.empty((rows, n_out), dtype=np.int32)
    pos_out = np.empty((rows, n_out), dtype=np.int32)
    rc = lib().oracle_csm(kb.ctypes.data, vb.ctypes.data, kd, dg.ctypes.data, rows, N, D, n_sink, window, chunk,
                          float(ratio), best.ctypes.data, sim.ctypes.data, merged.ctypes.data, ko.ctypes.data,
                          vo.ctypes.data, deg_out.ctypes.data, pos_out.ctypes.data)
    _check(0 if rc == n_out else -1, "csm")
    # the buffers handed to C were views of k_out / v_out (bf16 through an int16 view)
    if k.dtype == torch.bfloat16:
        k_out = torch.from_numpy(ko).view(torch.bfloat16).reshape(k_out.shape)
        v_out = torch.from_numpy(vo).view(torch.bfloat16).reshape(v_out.shape)
    shp = lead if lead else ()
    return {"best": best.reshape(shp + (N,)), "sim": sim.reshape(shp + (N,)), "merged": merged.reshape(shp + (N,)),
            "k_out": k_out, "v_out": v_out, "deg_out": deg_out.reshape(shp + (n_out,)),
            "pos_out": pos_out.reshape(shp + (n_out,)), "m": m}


def centroid_attention(q, k, v, deg=None) -> np.ndarray:
    """Decode attention (fp64) of q [B, Hq, nq, D] over a cache k, v [B, Hkv, n, D] whose
    degrees deg [B, Hkv, n] (None: all 1) add ln(deg) to the logits.  Returns
    [B, Hq, nq, D] float64."""
    qb, qd = _as_buffer(q)
    kb, kd = _as_buffer(k)
    vb, vd = _as_buffer(v)
    assert kd == vd
    B, Hq, nq, D = q.shape
    _, Hkv, n, _ = k.shape
    dg = None if deg is None else np.ascontiguousarray(np.asarray(deg, dtype=np.int32).reshape(B, Hkv, n))
    out = np.empty((B, Hq, nq, D), dtype=np.float64)
    rc = lib().oracle_centroid_attention(qb.ctypes.data, qd, kb.ctypes.data, vb.ctypes.data, kd,
                                         None if dg is None else dg.ctypes.data, B, Hq, Hkv, nq, n, D,
                                         out.ctypes.data)
    _check(rc, "centroid_attention")
    return out


def compress(q, k, v, *, window: int, n_sink: int, pool_kernel: int, kv_budget: int,
             scope: int = SCOPE_PER_KV_HEAD, tsp_rate: float = 0.0, hidden=None,
             threads: int = 0) -> dict:
    """The whole path in fp64.

    q [L, B, Hq, w, D], k [L, B, Hkv, N, D]: scored over all L layers (and, for scope
    ALL_HEADS, over all heads).  v [B, Hkv, N, D] belongs to the last layer; the kept rows
    of the last layer's K and of v form the compact cache.  With tsp_rate > 0 the
    head-summed scores select the hidden-state rows that are propagated (TSP); that
    selection has its own budget (decoupled from kv_budget).
    """
    if q.dim() == 4:
        q, k = q.unsqueeze(0), k.unsqueeze(0)
    N = k.shape[3]
    lo, hi = n_sink, N - window
    s = score(q, k, window=window, scope=scope, threads=threads)
    pooled = pool(s, lo, hi, pool_kernel)
    idx = select(pooled, n_sink, window, kv_budget)
    k_last = k[-1]
    out = {"scores": s, "pooled": pooled, "idx": idx,
           "k_out": gather(k_last, idx), "v_out": gather(v, idx)}
    if tsp_rate > 0:
        n_tsp = tsp_count(N, window, n_sink, tsp_rate)
        B, H = s.shape[0], s.shape[1]
        s_all = s if H == 1 else accumulate(np.zeros((B, 1, N)), s)
        p_all = pool(s_all, lo, hi, pool_kernel)
        tidx = select(p_all, n_sink, window, n_tsp)
        out.update(tsp_scores=s_all, tsp_pooled=p_all, tsp_idx=tidx)
        if hidden is not None:
            out["hidden_out"] = gather(hidden.unsqueeze(1), tidx)[:, 0]
    return out
