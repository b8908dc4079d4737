"""ctypes binding of libkvc.so (include/kvc.h).

Argument marshalling only: every step of the compaction runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.  Importing this module
loads the in-tree libkvc.so (with KVC_CHECKS=1 in the environment: the range-checking build
libkvc_checks.so) and raises if it is missing; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
CHECKS = os.environ.get("KVC_CHECKS", "0") == "1"
LIB_PATH = os.path.join(_PKG, "libkvc_checks.so" if CHECKS else "libkvc.so")

KVC_OK, KVC_ERR_ARG, KVC_ERR_UNSUPPORTED, KVC_ERR_BUDGET, KVC_ERR_ALIGN = 0, 1, 2, 3, 4
KVC_ERR_WORKSPACE, KVC_ERR_CUDA, KVC_ERR_TIMEOUT, KVC_ERR_INDEX, KVC_ERR_CHECK = 5, 6, 7, 8, 9
KVC_F32, KVC_BF16 = 0, 1
KVC_SCOPE_PER_KV_HEAD, KVC_SCOPE_ALL_HEADS = 0, 1
KVC_FLAG_SIMT_SCORE = 1
KVC_FLAG_INJECT_WAIT_TIMEOUT = 2
KVC_STAGE_SCORE, KVC_STAGE_SELECT, KVC_STAGE_GATHER, KVC_STAGE_COUNT = 0, 1, 2, 3

EXPORTED = ("kvc_workspace_size", "kvc_score", "kvc_accumulate", "kvc_pool", "kvc_topk_workspace_size",
            "kvc_topk", "kvc_gather", "kvc_compress", "kvc_tsp_count", "kvc_poll_error",
            "kvc_status_string", "kvc_version", "kvc_launch_count", "kvc_score_noalloc", "kvc_score_entropy",
            "kvc_row_stats", "kvc_csm_merges", "kvc_csm_ratio", "kvc_csm_workspace_size", "kvc_csm", "kvc_append",
            "kvc_decode_attention_workspace_size", "kvc_decode_attention", "kvc_shard_workspace_size",
            "kvc_shard_stats", "kvc_shard_scores", "kvc_select_hist", "kvc_select_emit", "kvc_select_pick",
            "kvc_select_ties", "kvc_select_kept", "kvc_checks_enabled")


class KvcError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {kvc_status_string(status)} (status {status})")


class Params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("N", ctypes.c_int32),
        ("D", ctypes.c_int32), ("window", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("n_sink", ctypes.c_int32), ("pool_kernel", ctypes.c_int32), ("kv_budget", ctypes.c_int32),
        ("scope", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("tsp_rate", ctypes.c_float),
        ("hidden_dim", ctypes.c_int32), ("spin_limit", ctypes.c_int64), ("flags", ctypes.c_uint32),
        ("reserved", ctypes.c_uint32), ("stage_events", ctypes.POINTER(ctypes.c_void_p)),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m long_context_kv_kvc_b200.build"
                          f"{' --checks' if CHECKS else ''}`")
    L = ctypes.CDLL(LIB_PATH)
    P, vp, i32, sz, st = ctypes.POINTER(Params), ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_int
    sig = {
        "kvc_workspace_size": (st, [P, ctypes.POINTER(sz)]),
        "kvc_score": (st, [P, vp, vp, vp, vp, sz, vp]),
        "kvc_accumulate": (st, [vp, vp, i32, i32, i32, i32, vp]),
        "kvc_pool": (st, [vp, vp, i32, i32, i32, i32, i32, i32, vp]),
        "kvc_topk_workspace_size": (st, [i32, i32, i32, ctypes.POINTER(sz)]),
        "kvc_topk": (st, [vp, i32, i32, i32, i32, i32, i32, vp, vp, sz, vp]),
        "kvc_gather": (st, [vp, i32, i32, i32, sz, vp, i32, i32, vp, vp]),
        "kvc_compress": (st, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "kvc_tsp_count": (i32, [i32, i32, i32, ctypes.c_float]),
        "kvc_poll_error": (st, [vp]),
        "kvc_status_string": (ctypes.c_char_p, [st]),
        "kvc_version": (ctypes.c_char_p, []),
        "kvc_launch_count": (ctypes.c_uint64, []),
        "kvc_score_noalloc": (st, [P, vp, vp, vp, vp]),
        "kvc_score_entropy": (st, [P, vp, vp, vp, vp, vp, sz, vp]),
        "kvc_row_stats": (st, [vp, i32, i32, i32, i32, vp, i32, vp, vp, vp]),
        "kvc_csm_merges": (i32, [i32, i32, i32, i32, ctypes.c_float]),
        "kvc_csm_ratio": (ctypes.c_float, [ctypes.c_float, ctypes.c_float, i32]),
        "kvc_csm_workspace_size": (st, [i32, i32, i32, i32, i32, i32, ctypes.c_float, ctypes.POINTER(sz)]),
        "kvc_csm": (st, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, i32, ctypes.c_float, vp, vp, vp, vp,
                         i32, vp, sz, vp]),
        "kvc_append": (st, [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, i32, i32, i32, i32, vp]),
        "kvc_decode_attention_workspace_size": (st, [i32, i32, i32, i32, i32, ctypes.POINTER(sz)]),
        "kvc_decode_attention": (st, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, sz, vp]),
        "kvc_shard_workspace_size": (st, [P, i32, ctypes.POINTER(sz)]),
        "kvc_shard_stats": (st, [P, vp, vp, i32, i32, vp, vp, sz, vp]),
        "kvc_shard_scores": (st, [P, vp, vp, i32, i32, vp, i32, vp, vp, sz, vp]),
        "kvc_select_hist": (st, [vp, i32, i32, i32, i32, vp, i32, i32, vp, vp]),
        "kvc_select_emit": (st, [vp, i32, i32, i32, i32, vp, vp, i32, vp, i32, vp, vp]),
        "kvc_select_pick": (st, [vp, vp, i32, i32, i32, vp, vp, vp, vp]),
        "kvc_select_ties": (st, [vp, i32, i32, i32, vp, vp, vp]),
        "kvc_select_kept": (st, [vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]),
        "kvc_checks_enabled": (i32, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    return L


lib = _load()


# ----------------------------------------------------------------------------- helpers

def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(st: int, what: str):
    if st != KVC_OK:
        raise KvcError(st, what)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return KVC_F32
    if dt == torch.bfloat16:
        return KVC_BF16
    raise ValueError(f"unsupported dtype {dt}")


def make_params(*, B, Hq, Hkv, N, window, dtype, n_sink=1, pool_kernel=7, kv_budget, D=128,
                scope=KVC_SCOPE_PER_KV_HEAD, n_layers=1, tsp_rate=0.0, hidden_dim=0, spin_limit=0,
                flags=0) -> Params:
    p = Params()
    p.B, p.Hq, p.Hkv, p.N, p.D, p.window = B, Hq, Hkv, N, D, window
    p.dtype = dtype if isinstance(dtype, int) else dtype_code(dtype)
    p.n_sink, p.pool_kernel, p.kv_budget, p.scope, p.n_layers = n_sink, pool_kernel, kv_budget, scope, n_layers
    p.tsp_rate, p.hidden_dim, p.spin_limit, p.flags, p.reserved = tsp_rate, hidden_dim, spin_limit, flags, 0
    p.stage_events = None
    return p


def params_for(wl, **overrides) -> Params:
    """Parameters of a synth.Workload (same field names)."""
    kw = dict(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, N=wl.N, D=wl.D, window=wl.window,
              dtype=KVC_F32 if wl.dtype == "f32" else KVC_BF16, n_sink=wl.n_sink,
              pool_kernel=wl.pool_kernel, kv_budget=wl.kv_budget, scope=wl.scope,
              n_layers=wl.n_layers, tsp_rate=wl.tsp_rate, hidden_dim=wl.hidden_dim)
    kw.update(overrides)
    return make_params(**kw)


# ------------------------------------------------------------------------ entry points

def kvc_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.kvc_workspace_size(ctypes.byref(p), ctypes.byref(n)), "kvc_workspace_size")
    return n.value


def kvc_score(p: Params, q, k, scores, ws, stream=None):
    _check(lib.kvc_score(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(scores), _ptr(ws),
                         ws.numel() * ws.element_size(), _stream(stream)), "kvc_score")


def kvc_score_noalloc(p: Params, q, k, scores, stream=None):
    """kvc_score without a workspace, for callers that cannot allocate device memory; the
    library's fixed 4 MiB per-device scratch array stands in for it (see include/kvc.h)."""
    _check(lib.kvc_score_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(scores), _stream(stream)),
           "kvc_score_noalloc")


def kvc_score_entropy(p: Params, q, k, scores, entropy, ws, stream=None):
    """kvc_score plus the attention entropy (nats) of every window query row, in one pass;
    entropy is [n_layers, B, Hq, window] fp32."""
    _check(lib.kvc_score_entropy(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(scores), _ptr(entropy), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)), "kvc_score_entropy")


def kvc_row_stats(scores, n_sink, window, cand_var, idx=None, kept_mass=None, stream=None):
    """Per score row of scores [..., N]: population variance over [n_sink, N - window) into
    cand_var, and (with idx [..., budget]) the share of the row's mass at idx into kept_mass."""
    N = scores.shape[-1]
    rows = scores.numel() // N
    budget = idx.shape[-1] if idx is not None else 0
    _check(lib.kvc_row_stats(_ptr(scores), rows, N, n_sink, window, _ptr(idx) if idx is not None else None,
                             budget, _ptr(kept_mass) if kept_mass is not None else None, _ptr(cand_var),
                             _stream(stream)), "kvc_row_stats")


def kvc_csm_merges(N, n_sink, window, chunk, ratio) -> int:
    m = int(lib.kvc_csm_merges(N, n_sink, window, chunk, ratio))
    if m < 0:
        raise KvcError(KVC_ERR_ARG, "kvc_csm_merges: invalid arguments")
    return m


def kvc_csm_ratio(r_init, delta, round_) -> float:
    return float(lib.kvc_csm_ratio(r_init, delta, round_))


def kvc_csm_workspace_size(B, H, N, n_sink, window, chunk, ratio) -> int:
    nb = ctypes.c_size_t(0)
    _check(lib.kvc_csm_workspace_size(B, H, N, n_sink, window, chunk, ratio, ctypes.byref(nb)), "kvc_csm_workspace_size")
    return nb.value


def kvc_csm(k, v, n_sink, window, chunk, ratio, deg=None, out=None, ws=None, stream=None, n=None, pos=None,
            ld_out=None) -> dict:
    """One Chunked Soft Matching round over the first n (default: all) rows of k, v
    [B, H, cap, D]; returns (and fills, when given as `out`) k_out, v_out [B, H, cap_out, D],
    deg_out and pos_out [B, H, cap_out] whose first N - m rows are the kept tokens.  deg and
    pos (nullable) share k's row layout; without `out` the outputs are dense (cap_out =
    N - m) unless ld_out is given."""
    B, H, cap, D = k.shape
    if v.dtype != k.dtype or v.shape != k.shape:
        raise KvcError(KVC_ERR_ARG, "kvc_csm: k and v must have the same shape and dtype")
    N = cap if n is None else n
    dt = KVC_BF16 if k.dtype == torch.bfloat16 else KVC_F32
    m = kvc_csm_merges(N, n_sink, window, chunk, ratio)
    if out is None:
        co = N - m if ld_out is None else ld_out
        out = {"k_out": torch.empty((B, H, co, D), dtype=k.dtype, device=k.device),
               "v_out": torch.empty((B, H, co, D), dtype=k.dtype, device=k.device),
               "deg_out": torch.empty((B, H, co), dtype=torch.int32, device=k.device),
               "pos_out": torch.empty((B, H, co), dtype=torch.int32, device=k.device)}
    cap_out = out["k_out"].shape[2]
    if ws is None:
        ws = torch.empty(max(kvc_csm_workspace_size(B, H, N, n_sink, window, chunk, ratio), 256), dtype=torch.uint8,
                         device=k.device)
    _check(lib.kvc_csm(_ptr(k), _ptr(v), _ptr(deg) if deg is not None else None,
                       _ptr(pos) if pos is not None else None, B, H, N, cap, D, dt, n_sink, window, chunk, ratio,
                       _ptr(out["k_out"]), _ptr(out["v_out"]), _ptr(out["deg_out"]), _ptr(out["pos_out"]), cap_out,
                       _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "kvc_csm")
    return out


def kvc_append(k_cache, v_cache, n, k_new, v_new, deg_cache=None, pos_cache=None, pos0=0, stream=None):
    """Writes k_new, v_new [B, H, t_new, D] into rows n .. n + t_new - 1 of the caches
    [B, H, cap, D] (degrees 1, positions pos0 ..)."""
    B, H, cap, D = k_cache.shape
    t_new = k_new.shape[2]
    if not (k_new.dtype == v_new.dtype == v_cache.dtype == k_cache.dtype):
        raise KvcError(KVC_ERR_ARG, "kvc_append: caches and new rows must share one dtype")
    dt = KVC_BF16 if k_cache.dtype == torch.bfloat16 else KVC_F32
    _check(lib.kvc_append(_ptr(k_cache), _ptr(v_cache), _ptr(deg_cache) if deg_cache is not None else None,
                          _ptr(pos_cache) if pos_cache is not None else None, B, H, cap, n, _ptr(k_new), _ptr(v_new),
                          t_new, pos0, D, dt, _stream(stream)), "kvc_append")


def kvc_decode_attention_workspace_size(B, Hq, Hkv, nq, n) -> int:
    nb = ctypes.c_size_t(0)
    _check(lib.kvc_decode_attention_workspace_size(B, Hq, Hkv, nq, n, ctypes.byref(nb)),
           "kvc_decode_attention_workspace_size")
    return nb.value


def kvc_decode_attention(q, k, v, deg=None, n=None, out=None, ws=None, stream=None):
    """Attention of q [B, Hq, nq, D] over the first n (default: all) rows of the cache
    k, v [B, Hkv, cap, D] with ln(deg) added to the logits (deg [B, Hkv, cap] or None);
    returns out [B, Hq, nq, D] fp32."""
    B, Hq, nq, D = q.shape
    _, Hkv, cap, _ = k.shape
    if q.dtype != k.dtype or v.dtype != k.dtype or v.shape != k.shape:
        raise KvcError(KVC_ERR_ARG, "kvc_decode_attention: q, k and v must share one dtype; k and v one shape")
    n = cap if n is None else n
    dt = KVC_BF16 if k.dtype == torch.bfloat16 else KVC_F32
    if out is None:
        out = torch.empty((B, Hq, nq, D), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = torch.empty(max(kvc_decode_attention_workspace_size(B, Hq, Hkv, nq, n), 256), dtype=torch.uint8,
                         device=q.device)
    _check(lib.kvc_decode_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(deg) if deg is not None else None, B, Hq, Hkv,
                                    nq, n, cap, D, dt, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                    _stream(stream)), "kvc_decode_attention")
    return out


def kvc_shard_workspace_size(p, n_local) -> int:
    nb = ctypes.c_size_t(0)
    _check(lib.kvc_shard_workspace_size(ctypes.byref(p), n_local, ctypes.byref(nb)), "kvc_shard_workspace_size")
    return nb.value


def kvc_shard_stats(p, q, k_local, key_offset, ml, ws, stream=None):
    n_local = k_local.shape[-2]
    _check(lib.kvc_shard_stats(ctypes.byref(p), _ptr(q), _ptr(k_local), n_local, key_offset, _ptr(ml), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)), "kvc_shard_stats")


def kvc_shard_scores(p, q, k_local, key_offset, ml_all, scores, ws, stream=None):
    n_local = k_local.shape[-2]
    _check(lib.kvc_shard_scores(ctypes.byref(p), _ptr(q), _ptr(k_local), n_local, key_offset, _ptr(ml_all),
                                ml_all.shape[0], _ptr(scores), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)), "kvc_shard_scores")


def kvc_select_hist(pooled, lo, hi, prefix, prefix_bits, digit_bits, hist, stream=None):
    rows, n = pooled.shape[0] * pooled.shape[1], pooled.shape[-1]
    _check(lib.kvc_select_hist(_ptr(pooled), rows, n, lo, hi, _ptr(prefix), prefix_bits, digit_bits, _ptr(hist),
                               _stream(stream)), "kvc_select_hist")


def kvc_select_emit(pooled, lo, hi, thr, ties, pos_offset, out, count, stream=None):
    rows, n = pooled.shape[0] * pooled.shape[1], pooled.shape[-1]
    _check(lib.kvc_select_emit(_ptr(pooled), rows, n, lo, hi, _ptr(thr), _ptr(ties), pos_offset, _ptr(out),
                               out.shape[-1], _ptr(count), _stream(stream)), "kvc_select_emit")


def _int32(*ts):
    for t in ts:
        if t.dtype != torch.int32:
            raise TypeError(f"expected int32 tensors, got {t.dtype}")


def kvc_select_pick(hist, hist_local, prefix_bits, need, prefix, eq_local, stream=None):
    _int32(hist, hist_local, need, prefix, eq_local)
    rows, nb = hist.shape
    digit_bits = nb.bit_length() - 1
    _check(lib.kvc_select_pick(_ptr(hist), _ptr(hist_local), rows, digit_bits, prefix_bits, _ptr(need), _ptr(prefix),
                               _ptr(eq_local), _stream(stream)), "kvc_select_pick")


def kvc_select_ties(eq_all, rank, need, take, stream=None):
    _int32(eq_all, need, take)
    n_shards, rows = eq_all.shape
    _check(lib.kvc_select_ties(_ptr(eq_all), n_shards, rank, rows, _ptr(need), _ptr(take), _stream(stream)),
           "kvc_select_ties")


def kvc_select_kept(sel, count_sel, N, n_sink, window, key_offset, n_local, pos, local_idx, count, stream=None):
    _int32(sel, count_sel, pos, local_idx, count)
    rows, cap_sel = sel.shape
    _check(lib.kvc_select_kept(_ptr(sel), _ptr(count_sel), rows, cap_sel, N, n_sink, window, key_offset, n_local,
                               pos.shape[-1], _ptr(pos), _ptr(local_idx), _ptr(count), _stream(stream)),
           "kvc_select_kept")


def kvc_accumulate(acc, src, stream=None):
    B, Ho, N = acc.shape
    Hi = src.shape[1]
    _check(lib.kvc_accumulate(_ptr(acc), _ptr(src), B, Hi, Ho, N, _stream(stream)), "kvc_accumulate")


def kvc_pool(inp, out, lo, hi, kernel, stream=None):
    B, H, N = inp.shape
    _check(lib.kvc_pool(_ptr(inp), _ptr(out), B, H, N, lo, hi, kernel, _stream(stream)), "kvc_pool")


def kvc_topk_workspace_size(B, H, N) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.kvc_topk_workspace_size(B, H, N, ctypes.byref(n)), "kvc_topk_workspace_size")
    return n.value


def kvc_topk(pooled, n_sink, window, budget, idx, ws=None, stream=None):
    B, H, N = pooled.shape
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.kvc_topk(_ptr(pooled), B, H, N, n_sink, window, budget, _ptr(idx), _ptr(ws), nb,
                        _stream(stream)), "kvc_topk")


def kvc_gather(src, idx, dst, stream=None):
    """src [B, Hsrc, N, ...] -> dst [B, Hsrc, K, ...] via idx [B, Hidx, K]."""
    B, Hsrc, N = src.shape[:3]
    row_bytes = src[0, 0, 0].numel() * src.element_size() if src.dim() > 3 else src.element_size()
    Hidx, K = idx.shape[1], idx.shape[2]
    _check(lib.kvc_gather(_ptr(src), B, Hsrc, N, row_bytes, _ptr(idx), Hidx, K, _ptr(dst),
                          _stream(stream)), "kvc_gather")


def kvc_compress(p: Params, q, k, v, k_out, v_out, idx_out, hidden=None, hidden_out=None,
                 tsp_idx_out=None, ws=None, stream=None):
    _check(lib.kvc_compress(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(k_out), _ptr(v_out),
                            _ptr(idx_out), _ptr(hidden), _ptr(hidden_out), _ptr(tsp_idx_out), _ptr(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "kvc_compress")


def kvc_tsp_count(N, window, n_sink, rate) -> int:
    return int(lib.kvc_tsp_count(N, window, n_sink, float(rate)))


def kvc_poll_error(stream=None) -> int:
    return int(lib.kvc_poll_error(_stream(stream)))


def kvc_checks_enabled() -> bool:
    return bool(lib.kvc_checks_enabled())


def kvc_status_string(st: int) -> str:
    return lib.kvc_status_string(st).decode()


def kvc_launch_count() -> int:
    return int(lib.kvc_launch_count())


def kvc_version() -> str:
    return lib.kvc_version().decode()


# ------------------------------------------------------------------ convenience front

def output_shapes(p: Params) -> dict:
    Hs = p.Hkv if p.scope == KVC_SCOPE_PER_KV_HEAD else 1
    shapes = {"k_out": (p.B, p.Hkv, p.kv_budget, p.D), "v_out": (p.B, p.Hkv, p.kv_budget, p.D),
              "idx_out": (p.B, Hs, p.kv_budget)}
    if p.tsp_rate > 0:
        n = kvc_tsp_count(p.N, p.window, p.n_sink, p.tsp_rate)
        shapes.update(tsp_idx_out=(p.B, 1, n), hidden_out=(p.B, n, p.hidden_dim))
    return shapes


class Compressor:
    """Holds the workspace and output buffers of one parameter set; `__call__` runs the
    whole path through kvc_compress.  Inputs on the host are copied to the device and the
    outputs copied back (the end-to-end form); device inputs are used in place."""

    def __init__(self, p: Params, device="cuda"):
        self.p = p
        self.device = torch.device(device)
        td = torch.float32 if p.dtype == KVC_F32 else torch.bfloat16
        self.ws = torch.empty(max(kvc_workspace_size(p), 256), dtype=torch.uint8, device=self.device)
        self.out = {}
        for name, shape in output_shapes(p).items():
            dt = torch.int32 if name.endswith("idx_out") else td
            self.out[name] = torch.empty(shape, dtype=dt, device=self.device)

    def run_device(self, q, k, v, hidden=None, stream=None):
        o = self.out
        kvc_compress(self.p, q, k, v, o["k_out"], o["v_out"], o["idx_out"], hidden, o.get("hidden_out"),
                     o.get("tsp_idx_out"), self.ws, stream)
        return o

    def __call__(self, q, k, v, hidden=None, stream=None):
        if q.is_cuda:
            return self.run_device(q, k, v, hidden, stream)
        dev = [t.to(self.device, non_blocking=True) if t is not None else None for t in (q, k, v, hidden)]
        o = self.run_device(*dev, stream=stream)
        host = {name: t.to("cpu", non_blocking=True) for name, t in o.items()}
        (stream or torch.cuda.current_stream()).synchronize()
        return host
