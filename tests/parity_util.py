"""Comparison rules between the CUDA path and the fp64 oracle.

Scores: |s_gpu - s_ref| <= 1e-3 |s_ref| + 1e-30 at every position.
Index sets: with T the oracle's k_sel-th largest pooled candidate score, every candidate
with s~_ref > T (1 + 1e-3) must be kept and every one with s~_ref < T (1 - 1e-3) must not;
only candidates inside that band may differ.  The GPU tests use the tighter band of
error_band(): 2.5x the worst score error measured on the same case.  The count, the sinks, the window and the
ascending order are exact.  Gathered rows are bit-exact given the GPU's own indices.
Chunked Soft Matching rows: see check_csm_row.
"""
import numpy as np
import torch

from long_context_kv_kvc_b200 import synth
from oracle import oracle as O

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
    order = np.lexsort((np.arange(cand.size), -cand))  # score descending, ties to the lower position
    T = cand[order[k_sel - 1]]
    must = S + np.nonzero(cand > T * (1 + rtol))[0]
    mustnot = S + np.nonzero(cand < T * (1 - rtol))[0]
    missing = np.setdiff1d(must, sel)
    extra = np.intersect1d(mustnot, sel)
    assert missing.size == 0, f"{missing.size} clearly-above-threshold tokens dropped"
    assert extra.size == 0, f"{extra.size} clearly-below-threshold tokens kept"
    ref_sel = np.sort(S + np.array(order[:k_sel]))
    return bool(np.array_equal(ref_sel, sel))


def check_index_sets(idx, pooled_ref, N, S, w, budget, rtol=SCORE_RTOL):
    idx = np.asarray(idx)
    rows = idx.reshape(-1, budget)
    ref = pooled_ref.reshape(-1, N)
    exact = [check_index_row(rows[r], ref[r], N, S, w, budget, rtol=rtol) for r in range(rows.shape[0])]
    return sum(exact) / len(exact)


def error_band(worst_rel):
    """The band inside which the GPU's index set may differ from the oracle's, given the worst
    relative score error actually measured on the case: a pooled value carries at most that
    error, so two candidates can only trade places if they are within (1 + e) / (1 - e) of
    each other; 2.5 e covers it.  Never wider than the contract's 1e-3, never below 1e-6."""
    return float(min(SCORE_RTOL, max(2.5 * worst_rel, 1e-6)))


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


CSM_BAND = 1e-5  # cosine band inside which fp32 (GPU) and fp64 (oracle) merge decisions may differ


def check_csm_row(kr, vr, dr, out_k, out_v, out_d, out_p, S, w, chunk, ratio, dtype):
    """One Chunked Soft Matching row against the oracle: the band rule (CSM_BAND) on the merge
    set, then every kept row given the GPU's merges (out_p: indices of the kept input rows)."""
    N = kr.shape[0]
    ref = O.csm(kr, vr, dr, n_sink=S, window=w, chunk=chunk, ratio=ratio)
    m = ref["m"]
    pos = np.asarray(out_p, dtype=np.int64)
    assert pos.size == N - m and np.all(np.diff(pos) > 0)
    is_merged = np.ones(N, dtype=bool)
    is_merged[pos] = False
    merged = np.nonzero(is_merged)[0]
    assert merged.size == m
    sim, best = ref["sim"], ref["best"]
    assert np.all(best[merged] >= 0), "a token without a match was merged"
    if m:
        T = np.sort(sim[best >= 0])[::-1][m - 1]
        must = (best >= 0) & (sim > T + CSM_BAND)
        mustnot = (best >= 0) & (sim < T - CSM_BAND)
        assert not np.any(must & ~is_merged), f"{int((must & ~is_merged).sum())} clearly better matches not merged"
        assert not np.any(mustnot & is_merged), "clearly worse matches merged"
    # the B token each merged A joins: the best match in fp64, unless the runner-up is within
    # the band (then neither candidate row is checked)
    kk, vv = kr.double().numpy(), vr.double().numpy()
    nrm = np.linalg.norm(kk, axis=1)
    unit = np.divide(kk, nrm[:, None], out=np.zeros_like(kk), where=nrm[:, None] > 0)
    owner = np.full(N, -1, dtype=np.int64)
    ambiguous = np.zeros(N, dtype=bool)
    for c0 in range(S, N - w, chunk):
        c1 = min(c0 + chunk, N - w)
        A = np.arange(c0, c1, 2)
        Bs = np.arange(c0 + 1, c1, 2)
        A = A[is_merged[A]]
        if A.size == 0 or Bs.size == 0:
            continue
        sm = unit[A] @ unit[Bs].T
        order = np.argsort(-sm, axis=1, kind="stable")
        owner[A] = Bs[order[:, 0]]
        if Bs.size > 1:
            gap = sm[np.arange(A.size), order[:, 0]] - sm[np.arange(A.size), order[:, 1]]
            close = gap < CSM_BAND
            ambiguous[Bs[order[close, 0]]] = True
            ambiguous[Bs[order[close, 1]]] = True
    # expected rows of the kept tokens: degree-weighted sums over the token and its absorbed ones
    d = np.asarray(dr, dtype=np.float64)
    n = d.copy()
    sk, sv = d[:, None] * kk, d[:, None] * vv
    ak, av = np.abs(sk), np.abs(sv)  # magnitude of the summands: the scale of the rounding error
    src = merged
    np.add.at(n, owner[src], d[src])
    np.add.at(sk, owner[src], d[src, None] * kk[src])
    np.add.at(sv, owner[src], d[src, None] * vv[src])
    np.add.at(ak, owner[src], d[src, None] * np.abs(kk[src]))
    np.add.at(av, owner[src], d[src, None] * np.abs(vv[src]))
    has = np.zeros(N, dtype=bool)
    has[owner[src]] = True
    check = ~ambiguous[pos]
    np.testing.assert_array_equal(np.asarray(out_d)[check], n[pos][check].astype(np.int64))
    single = check & ~has[pos]
    assert torch.equal(out_k[torch.from_numpy(single)], kr[torch.from_numpy(pos[single])]), "unmerged rows not copied"
    assert torch.equal(out_v[torch.from_numpy(single)], vr[torch.from_numpy(pos[single])]), "unmerged rows not copied"
    multi = check & has[pos]
    for s_, a_, got in ((sk, ak, out_k), (sv, av, out_v)):
        want = s_[pos[multi]] / n[pos[multi], None]
        scale = a_[pos[multi]] / n[pos[multi], None]
        g = got[torch.from_numpy(multi)].double().numpy()
        err = np.abs(g - want)
        # fp32 sums: error below ~2^-23 of the summands' magnitude; a bf16 output adds half a
        # unit in its last place (2^-8 of the value at most)
        bound = 2e-6 * scale + (2.0 ** -8 * np.abs(want) if dtype == torch.bfloat16 else 0.0) + 1e-30
        assert np.all(err <= bound), f"merged rows off by {(err / np.maximum(scale, 1e-30)).max():.2e} of their scale"
    # When the GPU merged exactly the oracle's tokens into the same owners (the common case),
    # its kept rows are also compared with the oracle's own outputs: the GPU rounds an fp32
    # mean once, the oracle an fp64 one, so bf16 rows may differ by one unit in the last
    # place of the oracle's value and fp32 rows by the fp32 summation error.  Returns the
    # fraction of elements that are bit-identical (None when the merge sets differ).
    if not (np.array_equal(pos, np.asarray(ref["pos_out"], dtype=np.int64)) and not ambiguous[pos].any()):
        return None
    np.testing.assert_array_equal(np.asarray(out_d, dtype=np.int64), np.asarray(ref["deg_out"], dtype=np.int64))
    same = total = 0
    for got, want_t, a_ in ((out_k, ref["k_out"], ak), (out_v, ref["v_out"], av)):
        g = got.double().numpy()
        want = want_t.double().numpy()
        if dtype == torch.bfloat16:
            mag = np.abs(want)
            ulp = np.where(mag > 0, 2.0 ** (np.floor(np.log2(np.where(mag > 0, mag, 1.0))) - 7), 2.0 ** -133)
            bound = ulp
        else:
            bound = 2e-6 * a_[pos] / n[pos, None] + 1e-30
        err = np.abs(g - want)
        assert np.all(err <= bound), "kept rows differ from the oracle's by more than the rounding allows"
        same += int(np.count_nonzero(g == want))
        total += g.size
    return same / total


def _dev(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def run_case(K, wl, flags=0):
    """One workload through kvc_compress and kvc_score (K: the kvc binding module) against
    the oracle on every score row: scores, index sets (band of error_band), gathers bit for
    bit, and the TSP selection and hidden-row gather when the workload has one."""
    inp = synth.make_inputs(wl)
    dev = _dev(inp)
    p = K.params_for(wl, flags=flags)
    comp = K.Compressor(p)
    out = comp(dev["q"], dev["k"], dev["v"], dev.get("hidden"))
    Hs = wl.Hkv if wl.scope == K.KVC_SCOPE_PER_KV_HEAD else 1
    scores = torch.empty((wl.B, Hs, wl.N), dtype=torch.float32, device="cuda")
    K.kvc_score(p, dev["q"], dev["k"], scores, comp.ws)
    assert K.kvc_poll_error() == K.KVC_OK
    ref = O.compress(inp["q"], inp["k"], inp["v"], window=wl.window, n_sink=wl.n_sink,
                     pool_kernel=wl.pool_kernel, kv_budget=wl.kv_budget, scope=wl.scope,
                     tsp_rate=float(np.float32(wl.tsp_rate)), hidden=inp["hidden"])
    worst = check_scores(scores.cpu().numpy(), ref["scores"])
    band = error_band(worst)
    exact = check_index_sets(out["idx_out"].cpu().numpy(), ref["pooled"], wl.N, wl.n_sink, wl.window,
                             wl.kv_budget, rtol=band)
    print(f"{wl.name}: worst score error {worst:.2e}, index band {band:.1e}, exact index sets {exact:.3f}")
    check_gather(out["k_out"], dev["k"][-1], out["idx_out"].cpu().numpy())
    check_gather(out["v_out"], dev["v"], out["idx_out"].cpu().numpy())
    if wl.tsp_rate > 0:
        n_tsp = K.kvc_tsp_count(wl.N, wl.window, wl.n_sink, wl.tsp_rate)
        tsp_exact = check_index_sets(out["tsp_idx_out"].cpu().numpy(), ref["tsp_pooled"], wl.N, wl.n_sink,
                                     wl.window, n_tsp, rtol=band)
        print(f"{wl.name}: exact TSP index sets {tsp_exact:.3f}")
        check_gather(out["hidden_out"].unsqueeze(1), dev["hidden"].unsqueeze(1),
                     out["tsp_idx_out"].cpu().numpy())
    return out, ref, scores
