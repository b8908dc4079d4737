"""Sequence sharding through the C ABI on one GPU: the ranks run as host threads that
share cuda:0 and exchange through an in-process collective (they wait for each other on
the host only; no kernel waits on another).

* kvc_shard_stats / kvc_shard_scores over blocks equal kvc_score of the whole sequence on
  the same path (tensor cores, and CUDA cores) within 1e-5 relative (the log-sum-exp is
  merged in another order), and the oracle within 1e-3;
* kvc_select_hist / kvc_select_emit / kvc_select_pick / kvc_select_ties / kvc_select_kept
  equal their numpy contract bit for bit (ties, -0.0);
* the sharded compaction's union of kept positions passes the band rule against the fp64
  oracle, and every rank's kept rows are its source rows.
"""
import threading

import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity_util import check_index_sets, check_scores

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_kv_kvc_b200 import build
    build.build()
    from long_context_kv_kvc_b200 import kvc
    torch.cuda.set_device(0)
    return kvc


class ThreadComm:
    def __init__(self, rank, world, shared):
        self.rank, self.world, self.sh = rank, world, shared

    def all_gather(self, t):
        self.sh["slots"][self.rank] = t
        self.sh["barrier"].wait()
        out = torch.stack([x.to(t.device) for x in self.sh["slots"]])
        self.sh["barrier"].wait()
        return out

    def all_reduce_sum(self, t):
        return self.all_gather(t).sum(dim=0)


def run_ranks(cuts, fn):
    world = len(cuts) - 1
    shared = {"slots": [None] * world, "barrier": threading.Barrier(world, timeout=120)}
    results, errors = [None] * world, []

    def body(r):
        try:
            results[r] = fn(ThreadComm(r, world, shared), cuts[r], cuts[r + 1])
        except Exception as e:  # surfaces in the main thread
            errors.append(e)
            shared["barrier"].abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    if errors:
        raise errors[0]
    return results


def order_key(x32):
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).copy()
    b[b == np.uint32(0x80000000)] = 0
    neg = (b & np.uint32(0x80000000)) != 0
    return np.where(neg, ~b, b | np.uint32(0x80000000)).astype(np.uint32)


@pytest.mark.parametrize("flags", [0, 1], ids=["tensor-cores", "cuda-cores"])
def test_shard_scores_match_whole_sequence(K, flags):
    from long_context_kv_kvc_b200 import synth
    wl = synth.scaled(synth.LLAMA8B_32K, B=2, Hq=8, Hkv=2, N=3001, kv_budget=300, n_hubs=16)
    inp = synth.make_inputs(wl, with_v=False, with_hidden=False)
    q, k = inp["q"][0].cuda(), inp["k"][0].cuda()
    p = K.params_for(wl, flags=flags)
    whole = torch.empty((wl.B, wl.Hkv, wl.N), device="cuda")
    ws = torch.empty(K.kvc_workspace_size(p), dtype=torch.uint8, device="cuda")
    K.kvc_score(p, q, k, whole, ws)
    cuts = [0, 700, 1500, 2990, 3001]  # the last block holds part of the window only
    U, nq = wl.B * wl.Hkv, wl.Hq // wl.Hkv * wl.window
    mls, blocks = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        kb = k[:, :, a:b].contiguous()
        wsb = torch.empty(K.kvc_shard_workspace_size(p, b - a), dtype=torch.uint8, device="cuda")
        ml = torch.empty((U, nq, 2), device="cuda")
        K.kvc_shard_stats(p, q, kb, a, ml, wsb)
        mls.append(ml)
        blocks.append((a, b, kb, wsb))
    ml_all = torch.stack(mls)
    parts = []
    for a, b, kb, wsb in blocks:
        s = torch.empty((wl.B, wl.Hkv, b - a), device="cuda")
        K.kvc_shard_scores(p, q, kb, a, ml_all, s, wsb)
        parts.append(s)
    assert K.kvc_poll_error() == K.KVC_OK
    got = torch.cat(parts, dim=2).cpu().numpy()
    check_scores(got, whole.cpu().numpy().astype(np.float64), rtol=1e-5)
    check_scores(got, O.score(inp["q"], inp["k"], window=wl.window))


def test_select_hist_and_emit_contract(K):
    g = np.random.default_rng(4)
    rows, n, lo, hi = 5, 3000, 7, 2960
    x = g.standard_normal((1, rows, n)).astype(np.float32)
    x[:, :, ::13] = np.float32(0.5)                 # exact ties
    x[:, :, 5::17] = np.float32(-0.0)
    x[:, :, 6::17] = np.float32(0.0)
    dev = torch.from_numpy(x).cuda()
    keys = order_key(x[0, :, lo:hi])
    for prefix_bits, digit_bits in [(0, 11), (11, 11), (22, 10), (3, 12)]:
        pre = keys[np.arange(rows), np.arange(rows) * 37]  # a key present in each row
        pre_t = torch.from_numpy(pre.view(np.int32).copy()).cuda()
        hist = torch.empty((rows, 1 << digit_bits), dtype=torch.int32, device="cuda")
        K.kvc_select_hist(dev, lo, hi, pre_t, prefix_bits, digit_bits, hist)
        want = np.zeros((rows, 1 << digit_bits), dtype=np.int64)
        for r in range(rows):
            kk = keys[r]
            if prefix_bits:
                kk = kk[(kk >> np.uint32(32 - prefix_bits)) == (pre[r] >> np.uint32(32 - prefix_bits))]
            want[r] = np.bincount(((kk >> np.uint32(32 - prefix_bits - digit_bits)) &
                                   np.uint32((1 << digit_bits) - 1)).astype(np.int64), minlength=1 << digit_bits)
        assert np.array_equal(hist.cpu().numpy(), want)
    thr = order_key(np.full(rows, 0.5, dtype=np.float32))
    ties = np.array([0, 1, 5, 1000, 3], dtype=np.int32)
    cap = hi - lo
    out = torch.full((rows, cap), -1, dtype=torch.int32, device="cuda")
    cnt = torch.empty(rows, dtype=torch.int32, device="cuda")
    K.kvc_select_emit(dev, lo, hi, torch.from_numpy(thr.view(np.int32).copy()).cuda(), torch.from_numpy(ties).cuda(),
                      -3, out, cnt)
    assert K.kvc_poll_error() == K.KVC_OK
    for r in range(rows):
        eq = keys[r] == thr[r]
        sel = (keys[r] > thr[r]) | (eq & (np.cumsum(eq) - 1 < ties[r]))
        want = -3 + lo + np.nonzero(sel)[0]
        assert cnt[r].item() == want.size
        assert np.array_equal(out[r, :want.size].cpu().numpy(), want)


def test_select_pick_ties_kept_contract(K):
    g = np.random.default_rng(5)
    rows = 6
    for digit_bits, prefix_bits in [(11, 0), (11, 11), (10, 22), (12, 3)]:
        nb = 1 << digit_bits
        hist_local = g.integers(0, 4, (rows, nb)).astype(np.int32)
        hist_local[:, ::7] = 0
        hist = hist_local + g.integers(0, 3, (rows, nb)).astype(np.int32)
        need = np.array([1, 5, 100, int(hist[3].sum()), 2, 33], dtype=np.int32)
        prefix = g.integers(0, 1 << 16, rows).astype(np.uint32) << np.uint32(32 - max(prefix_bits, 1)) \
            if prefix_bits else np.zeros(rows, np.uint32)
        d_need = torch.from_numpy(need.copy()).cuda()
        d_pre = torch.from_numpy(prefix.view(np.int32).copy()).cuda()
        d_eq = torch.empty(rows, dtype=torch.int32, device="cuda")
        K.kvc_select_pick(torch.from_numpy(hist).cuda(), torch.from_numpy(hist_local).cuda(), prefix_bits, d_need,
                          d_pre, d_eq)
        from_top = np.cumsum(hist[:, ::-1].astype(np.int64), axis=1)
        i = np.argmax(from_top >= need[:, None], axis=1)
        b = nb - 1 - i
        r = np.arange(rows)
        want_need = need - (from_top[r, i] - hist[r, b])
        want_pre = prefix | (b.astype(np.uint32) << np.uint32(32 - prefix_bits - digit_bits))
        assert np.array_equal(d_need.cpu().numpy(), want_need)
        assert np.array_equal(d_pre.cpu().numpy().view(np.uint32), want_pre)
        assert np.array_equal(d_eq.cpu().numpy(), hist_local[r, b])
    eq_all = g.integers(0, 5, (3, rows)).astype(np.int32)
    need = np.array([0, 1, 4, 7, 20, 3], dtype=np.int32)
    for rank in range(3):
        take = torch.empty(rows, dtype=torch.int32, device="cuda")
        K.kvc_select_ties(torch.from_numpy(eq_all).cuda(), rank, torch.from_numpy(need).cuda(), take)
        want = np.clip(need - eq_all[:rank].sum(axis=0), 0, eq_all[rank])
        assert np.array_equal(take.cpu().numpy(), want)
    # kept rows: sinks, selection, window of a block of the sequence
    N, S, w = 1000, 3, 16
    for key_off, n_local in [(0, 400), (400, 590), (990, 10), (2, 5)]:
        cap_sel = max(n_local, 1)
        sel = np.full((rows, cap_sel), -7, dtype=np.int32)
        # a block's selected positions are candidates: past the sinks, before the window
        cand = np.arange(max(S, key_off), min(N - w, key_off + n_local))
        cnt = g.integers(0, min(cand.size, 40) + 1, rows).astype(np.int32)
        for r_ in range(rows):
            sel[r_, :cnt[r_]] = np.sort(g.choice(cand, cnt[r_], replace=False))
        cap = min(n_local, 64)
        pos = torch.empty((rows, cap), dtype=torch.int32, device="cuda")
        local = torch.empty_like(pos)
        count = torch.empty(rows, dtype=torch.int32, device="cuda")
        K.kvc_select_kept(torch.from_numpy(sel).cuda(), torch.from_numpy(cnt).cuda(), N, S, w, key_off, n_local,
                          pos, local, count)
        sinks = [t for t in range(S) if key_off <= t < key_off + n_local]
        window = [t for t in range(N - w, N) if key_off <= t < key_off + n_local]
        over = False
        for r_ in range(rows):
            kept = sinks + sel[r_, :cnt[r_]].tolist() + window
            over |= len(kept) > cap
            assert count[r_].item() == len(kept)
            k_ = kept[:cap]
            assert pos[r_, :len(k_)].cpu().tolist() == k_
            assert np.all(pos[r_, len(k_):].cpu().numpy() == -1)
            assert local[r_, :len(k_)].cpu().tolist() == [t - key_off for t in k_]
        assert K.kvc_poll_error() == (K.KVC_ERR_INDEX if over else K.KVC_OK)


@pytest.mark.parametrize("cuts", [[0, 1000, 2001], [0, 3, 900, 1990, 2001]], ids=["2", "4-window-split"])
def test_sharded_compress_on_threads(K, cuts):
    from long_context_kv_kvc_b200 import synth
    from long_context_kv_kvc_b200.sharded import GpuOps, sharded_compress
    wl = synth.scaled(synth.LLAMA8B_32K, B=2, Hq=8, Hkv=2, N=2001, kv_budget=260, n_hubs=16)
    inp = synth.make_inputs(wl, with_hidden=False)
    q, k, v = inp["q"][0].cuda(), inp["k"][0].cuda(), inp["v"].cuda()
    p = K.params_for(wl)
    K.kvc_poll_error()  # the library's per-device state exists before the threads start
    torch.cuda.synchronize()

    def rank_fn(comm, a, b):
        return sharded_compress(comm, GpuOps(), p, q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(), a)

    res = run_ranks(cuts, rank_fn)
    torch.cuda.synchronize()
    assert K.kvc_poll_error() == K.KVC_OK
    rows = wl.B * wl.Hkv
    kept = [[] for _ in range(rows)]
    for r, out in enumerate(res):
        pos = out["pos"].cpu().numpy().reshape(rows, -1)
        cnt = out["count"].cpu().numpy().reshape(-1)
        for i in range(rows):
            b, h = divmod(i, wl.Hkv)
            kept[i].extend(pos[i, :cnt[i]].tolist())
            src = torch.from_numpy(pos[i, :cnt[i]]).long().cuda()
            assert torch.equal(out["k"][b, h, :cnt[i]], k[b, h, src])
            assert torch.equal(out["v"][b, h, :cnt[i]], v[b, h, src])
    idx = np.array(kept, dtype=np.int64).reshape(wl.B, wl.Hkv, -1)
    assert idx.shape[-1] == wl.kv_budget and np.all(np.diff(idx, axis=-1) > 0)
    ref_pooled = O.pool(O.score(inp["q"], inp["k"], window=wl.window), wl.n_sink, wl.N - wl.window, wl.pool_kernel)
    check_index_sets(idx, ref_pooled, wl.N, wl.n_sink, wl.window, wl.kv_budget)
