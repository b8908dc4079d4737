"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

No page prints a worked numerical example of the saliency path, so every pin here is a
closed form, an invariant, a special case that reduces to a textbook/library routine, or
brute force on a tiny input.  Each is chosen so that a plausible slip in the oracle (a
wrong logit scale, an off-by-one in the causal mask, a wrong GQA head mapping, a missing
max-shift, a reversed tie-break, a wrong pool radius or edge clipping) fails at least one.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

from oracle import oracle as O


def _zeros_case(B, Hq, Hkv, N, D, w, L=1):
    q = torch.randn(L, B, Hq, w, D, dtype=torch.float64, generator=torch.Generator().manual_seed(1))
    k = torch.zeros(L, B, Hkv, N, D, dtype=torch.float64)
    return q, k


def _uniform_closed_form(N, w, G):
    """All logits equal: query i (position N-w+i) spreads 1/(t_i+1) over keys 0..t_i."""
    s = np.zeros(N)
    for i in range(w):
        t = N - w + i
        s[: t + 1] += 1.0 / (t + 1)
    return G * s


@pytest.mark.parametrize("N,w,G", [(17, 3, 2), (40, 8, 4), (5, 5, 1)])
def test_all_equal_logits_closed_form(N, w, G):
    # K == 0 makes every logit 0; the softmax is then uniform over the visible keys.
    q, k = _zeros_case(1, 2 * G, 2, N, 16, w)
    s = O.score(q, k, window=w)
    ref = _uniform_closed_form(N, w, G)
    for h in range(2):
        np.testing.assert_allclose(s[0, h], ref, rtol=0, atol=1e-14)


def test_two_key_logistic_pins_scale():
    # One query at position 1 sees keys 0 and 1; with q = a e0 and k_j = b_j e0 the logits
    # are a b_j / sqrt(D), and the softmax of two logits is the logistic function.
    D = 16
    for a, b0, b1 in [(2.0, 3.0, -1.0), (0.5, -4.0, 6.0), (8.0, 1.0, 1.25)]:
        q = torch.zeros(1, 1, 1, 1, D, dtype=torch.float64)
        k = torch.zeros(1, 1, 1, 2, D, dtype=torch.float64)
        q[..., 0] = a
        k[0, 0, 0, 0, 0] = b0
        k[0, 0, 0, 1, 0] = b1
        s = O.score(q, k, window=1)
        x0, x1 = a * b0 / math.sqrt(D), a * b1 / math.sqrt(D)
        assert s[0, 0, 0] == pytest.approx(scipy.special.expit(x0 - x1), abs=1e-15)
        assert s[0, 0, 1] == pytest.approx(scipy.special.expit(x1 - x0), abs=1e-15)


def test_causal_mask_boundary():
    # The last key is visible to the last window query only: with equal logits it gets
    # exactly G / N, and the key before it gets G (1/(N-1) + 1/N) for w = 2.
    N, w, G = 9, 2, 3
    q, k = _zeros_case(1, G, 1, N, 8, w)
    s = O.score(q, k, window=w)[0, 0]
    assert s[N - 1] == pytest.approx(G / N, abs=1e-15)
    assert s[N - 2] == pytest.approx(G * (1 / (N - 1) + 1 / N), abs=1e-15)


def test_dominant_key_and_no_overflow():
    # One key with a logit gap >= 50 over all others takes all of the mass of every window
    # query that sees it.  Logits near 1000 also check that the max is subtracted
    # (exp(1000) overflows double).
    B, Hq, Hkv, N, D, w = 1, 4, 2, 64, 32, 4
    G = Hq // Hkv
    g = torch.Generator().manual_seed(3)
    k = torch.randn(1, B, Hkv, N, D, dtype=torch.float64, generator=g) * 0.01
    q = torch.zeros(1, B, Hq, w, D, dtype=torch.float64)
    q[..., 0] = 100.0
    k[..., 0] += 50.0  # all logits ~ 100*50/sqrt(32) ~ 884
    k[0, 0, :, 10, 0] = 60.0  # key 10 wins by ~177
    s = O.score(q, k, window=w)
    assert np.all(np.isfinite(s))
    np.testing.assert_allclose(s[0, :, 10], G * w, rtol=1e-12)
    assert s[0, :, np.arange(N) != 10].max() < 1e-60


def test_gqa_mapping_contiguous_groups():
    # q head g reads KV head g // G.  Heads 0,1 (group of KV head 0) have q = 0, so their
    # attention is uniform; heads 2,3 point at key 7 of KV head 1 with a huge gap.
    B, Hq, Hkv, N, D, w = 1, 4, 2, 30, 16, 3
    G = Hq // Hkv
    g = torch.Generator().manual_seed(5)
    k = torch.randn(1, B, Hkv, N, D, dtype=torch.float64, generator=g)
    q = torch.zeros(1, B, Hq, w, D, dtype=torch.float64)
    direction = k[0, 0, 1, 7] / k[0, 0, 1, 7].norm()
    q[0, 0, 2:] = 400.0 * direction
    s = O.score(q, k, window=w)
    np.testing.assert_allclose(s[0, 0], _uniform_closed_form(N, w, G), atol=1e-13)
    assert s[0, 1, 7] == pytest.approx(G * w, rel=1e-9)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mass_invariant(dtype):
    # Every window query distributes probability 1, so the scores of a KV head sum to G*w.
    B, Hq, Hkv, N, D, w = 2, 8, 2, 300, 128, 6
    g = torch.Generator().manual_seed(11)
    q = torch.randn(1, B, Hq, w, D, generator=g).to(dtype)
    k = torch.randn(1, B, Hkv, N, D, generator=g).to(dtype)
    s = O.score(q, k, window=w)
    np.testing.assert_allclose(s.sum(axis=-1), (Hq // Hkv) * w, rtol=1e-12)
    assert np.all(s >= 0)


def test_matches_library_softmax():
    # Cross-check against torch's float64 softmax (a library routine) with a causal mask.
    B, Hq, Hkv, N, D, w = 1, 6, 3, 50, 24, 5
    G = Hq // Hkv
    g = torch.Generator().manual_seed(7)
    q = torch.randn(1, B, Hq, w, D, dtype=torch.float64, generator=g) * 2
    k = torch.randn(1, B, Hkv, N, D, dtype=torch.float64, generator=g)
    s = O.score(q, k, window=w)
    pos = torch.arange(N - w, N)[:, None]
    mask = torch.arange(N)[None, :] > pos
    for h in range(Hkv):
        tot = torch.zeros(N, dtype=torch.float64)
        for gg in range(G):
            logits = q[0, 0, h * G + gg] @ k[0, 0, h].T / math.sqrt(D)
            tot += torch.softmax(logits.masked_fill(mask, -math.inf), dim=-1).sum(0)
        np.testing.assert_allclose(s[0, h], tot.numpy(), rtol=1e-12, atol=1e-15)


def test_layers_and_heads_are_sums():
    # StructKV's cumulative score is a plain sum over layers; ALL_HEADS sums KV heads.
    L, B, Hq, Hkv, N, D, w = 3, 2, 4, 2, 40, 16, 4
    g = torch.Generator().manual_seed(9)
    q = torch.randn(L, B, Hq, w, D, dtype=torch.float64, generator=g)
    k = torch.randn(L, B, Hkv, N, D, dtype=torch.float64, generator=g)
    s_all = O.score(q, k, window=w)
    s_sum = sum(O.score(q[l:l + 1], k[l:l + 1], window=w) for l in range(L))
    np.testing.assert_allclose(s_all, s_sum, rtol=1e-13)
    g_all = O.score(q, k, window=w, scope=O.SCOPE_ALL_HEADS)
    np.testing.assert_allclose(g_all[:, 0], s_all.sum(axis=1), rtol=1e-13)
    np.testing.assert_allclose(g_all.sum(axis=-1), L * Hq * w, rtol=1e-12)


def test_thread_count_does_not_change_result():
    g = torch.Generator().manual_seed(13)
    q = torch.randn(2, 2, 4, 4, 32, generator=g)
    k = torch.randn(2, 2, 2, 100, 32, generator=g)
    a = O.score(q, k, window=4, threads=1)
    b = O.score(q, k, window=4, threads=7)
    assert np.array_equal(a, b)


# ------------------------------------------------------------------------------ accumulate

def test_accumulate_group_sums():
    src = np.arange(2 * 6 * 5, dtype=np.float64).reshape(2, 6, 5)
    acc = np.ones((2, 3, 5))
    out = O.accumulate(acc.copy(), src)
    np.testing.assert_array_equal(out, 1 + src.reshape(2, 3, 2, 5).sum(axis=2))


# ------------------------------------------------------------------------------------ pool

@pytest.mark.parametrize("P", [1, 3, 7])
def test_pool_delta_gives_clipped_plateau(P):
    N, lo, hi = 30, 2, 25
    r = (P - 1) // 2
    for j0 in [lo, lo + 1, 12, hi - 2, hi - 1]:
        x = np.zeros((1, 1, N))
        x[0, 0, j0] = 1.0
        out = O.pool(x, lo, hi, P)[0, 0]
        want = np.zeros(N)
        want[max(lo, j0 - r): min(hi - 1, j0 + r) + 1] = 1.0
        np.testing.assert_array_equal(out, want)


def test_pool_ramp_and_no_leak_from_outside():
    N, lo, hi, P = 20, 3, 15, 5
    x = np.arange(N, dtype=np.float64)[None, None].copy()
    x[0, 0, lo - 1] = 1e9  # outside C: must not leak into pooled values
    x[0, 0, hi] = 1e9
    out = O.pool(x, lo, hi, P)[0, 0]
    for j in range(lo, hi):
        assert out[j] == min(hi - 1, j + 2)
    assert out[lo - 1] == 1e9 and out[hi] == 1e9  # pass-through outside C


def test_pool_matches_sliding_window_library():
    g = np.random.default_rng(0)
    x = g.random((2, 3, 57))
    lo, hi, P = 4, 50, 7
    r = P // 2
    out = O.pool(x, lo, hi, P)
    seg = np.pad(x[..., lo:hi], ((0, 0), (0, 0), (r, r)), constant_values=-np.inf)
    want = np.lib.stride_tricks.sliding_window_view(seg, P, axis=-1).max(axis=-1)
    np.testing.assert_array_equal(out[..., lo:hi], want)
    np.testing.assert_array_equal(out[..., :lo], x[..., :lo])
    np.testing.assert_array_equal(out[..., hi:], x[..., hi:])


# ---------------------------------------------------------------------------------- select

def _brute_force_selected(vals, k_sel):
    """Among all k_sel-subsets of candidate positions, the one with the largest multiset
    of values and, among those, the lexicographically smallest positions."""
    n = len(vals)
    best = None
    for comb in itertools.combinations(range(n), k_sel):
        key = (sorted((-vals[c] for c in comb)), comb)
        if best is None or key < best:
            best = key
    return list(best[1])


def test_select_brute_force_with_ties():
    g = np.random.default_rng(1)
    for trial in range(25):
        N, S, w = 14, 1, 2
        budget = S + w + int(g.integers(1, 6))
        vals = g.integers(0, 4, size=N).astype(np.float64)  # many ties
        idx = O.select(vals[None, None], S, w, budget)[0, 0]
        k_sel = budget - S - w
        sel = [S + c for c in _brute_force_selected(vals[S:N - w], k_sel)]
        want = sorted(list(range(S)) + sel + list(range(N - w, N)))
        assert list(idx) == want


def test_select_matches_library_sort_and_invariants():
    g = np.random.default_rng(2)
    B, H, N, S, w = 2, 3, 500, 4, 16
    vals = np.round(g.random((B, H, N)), 2)  # ties are common
    for budget in [S + w + 1, 60, 200, N]:
        idx = O.select(vals, S, w, budget)
        assert idx.shape == (B, H, budget)
        for b in range(B):
            for h in range(H):
                row = idx[b, h]
                assert np.all(np.diff(row) > 0)
                assert set(range(S)) <= set(row) and set(range(N - w, N)) <= set(row)
                ranked = sorted(range(S, N - w), key=lambda j: (-vals[b, h, j], j))
                sel = set(ranked[: budget - S - w])
                assert set(row) == sel | set(range(S)) | set(range(N - w, N))


def test_select_nested_in_budget_and_rejects_bad_budgets():
    g = np.random.default_rng(3)
    vals = g.random((1, 1, 200))
    prev = set()
    for budget in range(10, 200, 17):
        cur = set(O.select(vals, 2, 5, budget)[0, 0])
        assert prev <= cur
        prev = cur
    with pytest.raises(ValueError):
        O.select(vals, 2, 5, 7)  # budget < S + w + 1
    with pytest.raises(ValueError):
        O.select(vals, 2, 5, 201)  # budget > N


def test_select_all_equal_takes_lowest_indices():
    idx = O.select(np.ones((1, 1, 20)), 1, 3, 8)[0, 0]
    assert list(idx) == [0, 1, 2, 3, 4, 17, 18, 19]


# ---------------------------------------------------------------------------------- gather

def test_gather_is_a_row_copy():
    g = torch.Generator().manual_seed(4)
    src = torch.randn(2, 3, 40, 16, generator=g).to(torch.bfloat16)
    idx = np.stack([np.stack([np.sort(np.random.default_rng(b * 3 + h).choice(40, 7, replace=False))
                              for h in range(3)]) for b in range(2)]).astype(np.int32)
    out = O.gather(src, idx)
    for b in range(2):
        for h in range(3):
            assert torch.equal(out[b, h].view(torch.int16), src[b, h, idx[b, h]].view(torch.int16))
    shared = idx[:, :1]
    out1 = O.gather(src, shared)
    for h in range(3):
        assert torch.equal(out1[:, h], src[torch.arange(2)[:, None], h, torch.from_numpy(shared[:, 0]).long()])


# ------------------------------------------------------------------------------------- TSP

def test_tsp_count():
    assert O.tsp_count(65536, 32, 1, 0.2) == 13107 + 1 + 32
    assert O.tsp_count(100, 10, 1, 0.0) == 0
    assert O.tsp_count(100, 10, 1, 0.001) == 0  # floor(0.1) = 0 tokens
    assert O.tsp_count(100, 10, 1, 1.0) == 100  # capped at the 89 candidates


def test_compress_composition_invariants():
    g = torch.Generator().manual_seed(21)
    q = torch.randn(1, 2, 4, 4, 32, generator=g)
    k = torch.randn(1, 2, 2, 120, 32, generator=g)
    v = torch.randn(2, 2, 120, 32, generator=g)
    hidden = torch.randn(2, 120, 48, generator=g)
    out = O.compress(q, k, v, window=4, n_sink=1, pool_kernel=3, kv_budget=20, tsp_rate=0.25,
                     hidden=hidden)
    assert out["idx"].shape == (2, 2, 20)
    assert out["tsp_idx"].shape == (2, 1, 30 + 5)
    np.testing.assert_allclose(out["tsp_scores"][:, 0], out["scores"].sum(axis=1), rtol=1e-14)
    for b in range(2):
        assert torch.equal(out["hidden_out"][b], hidden[b, torch.from_numpy(out["tsp_idx"][b, 0]).long()])
        for h in range(2):
            assert torch.equal(out["k_out"][b, h], k[0, b, h, torch.from_numpy(out["idx"][b, h]).long()])


# ------------------------------------------------------------------- pivot metrics

@pytest.mark.parametrize("N,w,G", [(17, 3, 2), (40, 8, 4)])
def test_entropy_equal_logits_is_log_of_visible_count(N, w, G):
    # K == 0: every row's softmax is uniform over its t_i + 1 visible keys, so its entropy
    # is ln(t_i + 1) in nats (pins the mask, the normalisation and the natural log).
    q, k = _zeros_case(2, 2 * G, 2, N, 16, w, L=2)
    H = O.entropy(q, k, window=w)
    for i in range(w):
        np.testing.assert_allclose(H[..., i], math.log(N - w + i + 1), rtol=0, atol=1e-13)


def test_entropy_two_keys_is_binary_entropy():
    # One query seeing two keys with logits x0, x1: the binary entropy of expit(x0 - x1)
    # (pins the 1/sqrt(D) scale inside the entropy).
    D = 16
    for a, b0, b1 in [(2.0, 3.0, -1.0), (0.5, -4.0, 6.0), (8.0, 1.0, 1.25)]:
        q = torch.zeros(1, 1, 1, 1, D, dtype=torch.float64)
        k = torch.zeros(1, 1, 1, 2, D, dtype=torch.float64)
        q[..., 0] = a
        k[0, 0, 0, 0, 0] = b0
        k[0, 0, 0, 1, 0] = b1
        p = scipy.special.expit((a * b0 - a * b1) / math.sqrt(D))
        want = -(p * math.log(p) + (1 - p) * math.log(1 - p))
        assert O.entropy(q, k, window=1)[0, 0, 0, 0] == pytest.approx(want, abs=1e-14)


def test_entropy_dominant_key_is_zero_and_matches_library():
    # A key with a logit gap of ~1000 takes all the mass: entropy 0 (also pins the max
    # shift, exp(1000) overflows); random rows against torch's float64 softmax entropy.
    q = torch.zeros(1, 1, 2, 2, 8, dtype=torch.float64)
    k = torch.randn(1, 1, 1, 12, 8, dtype=torch.float64, generator=torch.Generator().manual_seed(5)) * 0.01
    q[..., 0] = 200.0
    k[0, 0, 0, 3, 0] = 40.0
    assert np.all(np.abs(O.entropy(q, k, window=2)) < 1e-12)
    g = torch.Generator().manual_seed(6)
    L, B, Hq, Hkv, N, D, w = 2, 2, 4, 2, 37, 16, 5
    q = torch.randn(L, B, Hq, w, D, dtype=torch.float64, generator=g)
    k = torch.randn(L, B, Hkv, N, D, dtype=torch.float64, generator=g)
    H = O.entropy(q, k, window=w)
    G = Hq // Hkv
    for layer in range(L):
        for b in range(B):
            for hq in range(Hq):
                x = q[layer, b, hq] @ k[layer, b, hq // G].T / math.sqrt(D)
                for i in range(w):
                    lp = torch.log_softmax(x[i, : N - w + i + 1], dim=0)
                    want = float(-(lp.exp() * lp).sum())
                    assert H[layer, b, hq, i] == pytest.approx(want, abs=1e-12)
    rows = np.array([0, 7, 31, L * B * Hq * w - 1], dtype=np.int32)
    np.testing.assert_array_equal(O.entropy(q, k, window=w, rows=rows), H.reshape(-1)[rows])


def test_row_stats_against_definitions():
    # kept mass against a brute-force sum; candidate variance against numpy's population
    # variance over [S, N - w); a constant row has variance 0; a full budget keeps mass 1.
    g = np.random.default_rng(8)
    B, H, N, S, w = 2, 3, 50, 2, 5
    s = g.random((B, H, N))
    idx = np.stack([np.sort(g.choice(N, 20, replace=False)) for _ in range(B * H)]).reshape(B, H, 20)
    km, cv = O.row_stats(s, S, w, idx)
    for b in range(B):
        for h in range(H):
            assert km[b, h] == pytest.approx(s[b, h, idx[b, h]].sum() / s[b, h].sum(), rel=1e-14)
            assert cv[b, h] == pytest.approx(np.var(s[b, h, S:N - w]), rel=1e-12)
    km_full, _ = O.row_stats(s, S, w, np.tile(np.arange(N, dtype=np.int32), (B, H, 1)))
    np.testing.assert_allclose(km_full, 1.0, rtol=1e-15)
    _, cv_const = O.row_stats(np.full((1, 1, N), 0.37), S, w)
    assert cv_const[0, 0] < 1e-30
    # variance over C only: values outside C do not move it
    s2 = s.copy()
    s2[..., :S] = 1e6
    s2[..., N - w:] = -1e6
    np.testing.assert_allclose(O.row_stats(s2, S, w)[1], cv, rtol=1e-13)


# ------------------------------------------------------------------- Chunked Soft Matching

def _csm_brute(k, deg, S, w, chunk, m, v=None):
    """Plain-Python restatement for tiny inputs: matches, the m merged A tokens, kept rows
    (of k, or of v when given, with k's matches)."""
    N = k.shape[0]
    kk = k.double().numpy()
    best, sim = {}, {}
    for c0 in range(S, N - w, chunk):
        c1 = min(c0 + chunk, N - w)
        A, B = list(range(c0, c1, 2)), list(range(c0 + 1, c1, 2))
        for a in A:
            if not B:
                continue
            sims = []
            for b in B:
                na, nb = np.linalg.norm(kk[a]), np.linalg.norm(kk[b])
                sims.append(float(kk[a] @ kk[b] / (na * nb)) if na > 0 and nb > 0 else 0.0)
            i = int(np.argmax(sims))  # first maximum: the lower position
            best[a], sim[a] = B[i], sims[i]
    order = sorted(best, key=lambda a: (-sim[a], a))
    merged = set(order[:m])
    src = kk if v is None else v.double().numpy()
    rows, degs, pos = [], [], []
    for j in range(N):
        if j in merged:
            continue
        parts = [j] + [a for a in sorted(merged) if best[a] == j]
        n = sum(int(deg[x]) for x in parts)
        rows.append(sum(int(deg[x]) * src[x] for x in parts) / n)
        degs.append(n)
        pos.append(j)
    return best, sim, merged, np.array(rows), np.array(degs), np.array(pos)


def test_csm_merge_count():
    # C = [1, 8) in chunks of 4: [1, 5) holds 2 A tokens, [5, 8) holds 2 -> 4 matchable
    assert O.csm_merges(10, 1, 2, 4, 0.5) == 3            # floor(0.5 * 7)
    assert O.csm_merges(10, 1, 2, 4, 0.25) == 1
    assert O.csm_merges(10, 1, 2, 4, 0.0) == 0
    assert O.csm_merges(9, 0, 0, 4, 0.5) == 4             # [0,4) [4,8) [8,9): the lone A is unmatchable
    assert O.csm_merges(5, 0, 0, 2, 0.5) == 2             # chunks [0,2) [2,4) [4,5)
    assert O.csm_ratio(0.5, 0.1, 0) == 0.5 and O.csm_ratio(0.5, 0.1, 2) == pytest.approx(0.3)
    assert O.csm_ratio(0.5, 0.2, 9) == 0.0


@pytest.mark.parametrize("N,S,w,chunk,r", [(23, 1, 3, 4, 0.5), (40, 0, 0, 6, 0.3), (31, 2, 5, 8, 0.45),
                                           (12, 1, 1, 2, 0.5)])
def test_csm_matches_brute_force(N, S, w, chunk, r):
    g = torch.Generator().manual_seed(N + chunk)
    k = torch.randn(N, 6, dtype=torch.float64, generator=g)
    k[S + 3] = 0.0  # a zero key: similarity 0 to everything
    v = torch.randn(N, 6, dtype=torch.float64, generator=g)
    deg = torch.randint(1, 5, (N,), generator=g).numpy().astype(np.int32)
    m = O.csm_merges(N, S, w, chunk, r)
    out = O.csm(k, v, deg, n_sink=S, window=w, chunk=chunk, ratio=r)
    best, sim, merged, rows, degs, pos = _csm_brute(k, deg, S, w, chunk, m)
    for a in range(N):
        if a in best:
            assert out["best"][a] == best[a] and out["sim"][a] == pytest.approx(sim[a], abs=1e-13)
        else:
            assert out["best"][a] == -1
    assert set(np.nonzero(out["merged"])[0].tolist()) == merged
    np.testing.assert_array_equal(out["pos_out"], pos)
    np.testing.assert_array_equal(out["deg_out"], degs)
    np.testing.assert_allclose(out["k_out"].numpy(), rows, rtol=1e-13, atol=1e-13)
    vrows = _csm_brute(k, deg, S, w, chunk, m, v=v)[3]
    np.testing.assert_allclose(out["v_out"].numpy(), vrows, rtol=1e-13, atol=1e-13)


def test_csm_invariants_and_closed_forms():
    # identical directions merge first (cosine 1); a B token absorbing an A token of the
    # same direction gives the degree-weighted mean; sinks, window and unmerged rows are
    # unchanged bit for bit; degrees are conserved; r = 0 is the identity
    N, D = 16, 8
    g = torch.Generator().manual_seed(21)
    k = torch.randn(N, D, dtype=torch.float32, generator=g)
    v = torch.randn(N, D, dtype=torch.float32, generator=g)
    k[5] = 2.0 * k[4]                      # chunk [4, 8) with S=0, chunk 4: A = {4, 6}, B = {5, 7}
    deg = np.array([1, 2, 1, 1, 3, 1, 2, 1, 1, 1, 4, 1, 1, 1, 1, 1], dtype=np.int32)
    out = O.csm(k, v, deg, n_sink=0, window=0, chunk=4, ratio=1 / 16)  # m = 1
    assert out["m"] == 1 and out["merged"][4] == 1 and out["best"][4] == 5
    assert out["sim"][4] == pytest.approx(1.0, abs=1e-7)
    j = list(out["pos_out"]).index(5)
    want = (3 * k[4].double() + 1 * k[5].double()) / 4
    np.testing.assert_allclose(out["k_out"][j].double().numpy(), want.numpy(), rtol=1e-6)
    assert out["deg_out"][j] == 4 and out["deg_out"].sum() == deg.sum()
    for o, p in enumerate(out["pos_out"]):
        if p != 5:
            assert torch.equal(out["k_out"][o], k[p]) and torch.equal(out["v_out"][o], v[p])
    ident = O.csm(k, v, deg, n_sink=2, window=3, chunk=4, ratio=0.0)
    assert torch.equal(ident["k_out"], k) and np.array_equal(ident["pos_out"], np.arange(N))
    big = O.csm(k, v, deg, n_sink=2, window=3, chunk=4, ratio=0.5)
    assert set(range(2)) <= set(big["pos_out"].tolist()) and set(range(N - 3, N)) <= set(big["pos_out"].tolist())
    assert big["deg_out"].sum() == deg.sum() and len(big["pos_out"]) == N - big["m"]
    assert np.all(np.diff(big["pos_out"]) > 0)


def test_csm_bf16_output_rounding():
    # merged rows are rounded to bf16 to nearest, ties to even: 1 and 1 + 2^-7 (degrees 1, 1)
    # average to 1 + 2^-8, a tie that rounds to 1; 1 and 1 + 3 * 2^-7 give 1 + 3 * 2^-8, which
    # rounds up to 1 + 2^-6
    D = 2
    for hi, want in [(1 + 2 ** -7, 1.0), (1 + 3 * 2 ** -7, 1 + 2 ** -6)]:
        k = torch.tensor([[1.0, 1.0], [hi, hi]], dtype=torch.bfloat16)
        out = O.csm(k, k, np.ones(2, np.int32), n_sink=0, window=0, chunk=2, ratio=0.5)
        assert out["m"] == 1 and out["k_out"].shape == (1, D)
        assert out["k_out"][0, 0].item() == want


def test_csm_ties_go_to_lower_position():
    # two B tokens with the same key: every A token of the chunk matches the lower one, and
    # equal similarities merge in position order
    a, b = [1.0, 0.2, 0.0], [0.3, 1.0, 0.5]
    k = torch.tensor([a, b, a, b, a, b, a, b], dtype=torch.float64)
    out = O.csm(k, k, np.ones(8, np.int32), n_sink=0, window=0, chunk=8, ratio=0.25)
    assert out["best"][0] == 1 and out["best"][2] == 1 and out["best"][4] == 1 and out["best"][6] == 1
    # all four A tokens tie; two merges take positions 0 and 2
    assert out["m"] == 2 and np.nonzero(out["merged"])[0].tolist() == [0, 2]


# ---------------------------------------------------------------- decode attention (CentroidKV sec. 4)

def _sdpa_gqa(q, k, v):
    """torch's float64 scaled-dot-product attention with each KV head serving its group."""
    G = q.shape[1] // k.shape[1]
    return torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double().repeat_interleave(G, dim=1), v.double().repeat_interleave(G, dim=1)).numpy()


@pytest.mark.parametrize("B,Hq,Hkv,nq,n,dtype", [(1, 4, 1, 1, 37, torch.float64), (2, 8, 2, 3, 70, torch.float32),
                                                  (1, 6, 3, 2, 129, torch.bfloat16)])
def test_centroid_attention_unit_degrees_is_library_attention(B, Hq, Hkv, nq, n, dtype):
    g = torch.Generator().manual_seed(n)
    q = torch.randn(B, Hq, nq, 128, generator=g).to(dtype)
    k = torch.randn(B, Hkv, n, 128, generator=g).to(dtype)
    v = torch.randn(B, Hkv, n, 128, generator=g).to(dtype)
    ref = _sdpa_gqa(q, k, v)
    np.testing.assert_allclose(O.centroid_attention(q, k, v), ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.centroid_attention(q, k, v, deg=np.ones((B, Hkv, n), np.int32)), ref, rtol=0,
                               atol=1e-12)


def test_centroid_attention_degree_is_replication():
    # a centroid of degree n attends exactly like n copies of itself with degree 1
    g = torch.Generator().manual_seed(5)
    B, Hq, Hkv, nq, n = 2, 4, 2, 2, 23
    q = torch.randn(B, Hq, nq, 128, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, n, 128, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, n, 128, generator=g, dtype=torch.float64)
    deg = torch.randint(1, 5, (B, Hkv, n), generator=g, dtype=torch.int32)
    got = O.centroid_attention(q, k, v, deg=deg.numpy())
    for b in range(B):
        for h in range(Hkv):
            reps = deg[b, h].long()
            kr = k[b, h].repeat_interleave(reps, dim=0)[None, None]
            vr = v[b, h].repeat_interleave(reps, dim=0)[None, None]
            want = O.centroid_attention(q[b:b + 1, 2 * h:2 * h + 2], kr, vr)
            np.testing.assert_allclose(got[b, 2 * h:2 * h + 2], want[0], rtol=0, atol=1e-12)


def test_centroid_attention_closed_forms():
    g = torch.Generator().manual_seed(9)
    q = torch.randn(1, 2, 1, 128, generator=g, dtype=torch.float64)
    # one cached row: the output is its value whatever the degree
    k1 = torch.randn(1, 1, 1, 128, generator=g, dtype=torch.float64)
    v1 = torch.randn(1, 1, 1, 128, generator=g, dtype=torch.float64)
    for d in (1, 7):
        np.testing.assert_allclose(O.centroid_attention(q, k1, v1, deg=np.full((1, 1, 1), d, np.int32)),
                                   v1.expand(1, 2, 1, 128).numpy(), rtol=0, atol=1e-14)
    # two rows: the weight of row 0 is the logistic function of the scaled logit gap plus
    # ln(n0 / n1)
    k2 = torch.randn(1, 1, 2, 128, generator=g, dtype=torch.float64)
    v2 = torch.randn(1, 1, 2, 128, generator=g, dtype=torch.float64)
    n0, n1 = 5, 2
    got = O.centroid_attention(q, k2, v2, deg=np.array([[[n0, n1]]], np.int32))
    for hq in range(2):
        gap = float((q[0, hq, 0] @ (k2[0, 0, 0] - k2[0, 0, 1])) / math.sqrt(128)) + math.log(n0 / n1)
        p0 = scipy.special.expit(gap)
        want = p0 * v2[0, 0, 0].numpy() + (1 - p0) * v2[0, 0, 1].numpy()
        np.testing.assert_allclose(got[0, hq, 0], want, rtol=0, atol=1e-13)
    # scaling every degree by the same factor changes nothing (softmax shift invariance)
    k = torch.randn(1, 1, 30, 128, generator=g, dtype=torch.float64)
    v = torch.randn(1, 1, 30, 128, generator=g, dtype=torch.float64)
    deg = torch.randint(1, 4, (1, 1, 30), generator=g, dtype=torch.int32).numpy()
    np.testing.assert_allclose(O.centroid_attention(q, k, v, deg=3 * deg), O.centroid_attention(q, k, v, deg=deg),
                               rtol=0, atol=1e-13)


def test_centroid_attention_gqa_groups():
    # KV head h holds the constant value h + 1: query head g must read KV head g // G
    g = torch.Generator().manual_seed(2)
    Hq, Hkv, n = 6, 3, 11
    q = torch.randn(1, Hq, 2, 128, generator=g, dtype=torch.float64)
    k = torch.randn(1, Hkv, n, 128, generator=g, dtype=torch.float64)
    v = (torch.arange(Hkv, dtype=torch.float64) + 1).view(1, Hkv, 1, 1).expand(1, Hkv, n, 128).contiguous()
    got = O.centroid_attention(q, k, v, deg=torch.randint(1, 9, (1, Hkv, n), generator=g).numpy())
    for hq in range(Hq):
        np.testing.assert_allclose(got[0, hq], hq // (Hq // Hkv) + 1.0, rtol=0, atol=1e-13)
