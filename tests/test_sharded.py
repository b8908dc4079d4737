"""Sequence sharding's host logic on CPU ranks (gloo): the exchanges, the pool halo, the
distributed radix select and the split of ties between ranks.

The steps on the data are numpy stand-ins with the kernels' contracts (fp32 scores, the
same order-preserving keys); the ranks' union of kept positions must match the unsharded
fp64 oracle under the band rule, every rank's kept rows must be its source rows, and the
result must not depend on how the sequence is cut into blocks.
"""
import os
import socket
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LOG2E = 1.4426950408889634


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def order_key(x32: np.ndarray) -> np.ndarray:
    """Monotone map of fp32 to uint32 (the kernels' contract; -0.0 reads as +0.0)."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).copy()
    b[b == np.uint32(0x80000000)] = 0
    neg = (b & np.uint32(0x80000000)) != 0
    return np.where(neg, ~b, b | np.uint32(0x80000000)).astype(np.uint32)


class NumpyOps:
    """fp64 arithmetic rounded to fp32 where the kernels store fp32."""

    def _logits(self, p, q, k_local, key_offset):
        q = q.double().numpy()
        k = k_local.double().numpy()
        B, Hq, w, D = q.shape
        Hkv, n = k.shape[1], k.shape[2]
        G = Hq // Hkv
        y = np.einsum("bhgwd,bhnd->bhgwn", q.reshape(B, Hkv, G, w, D), k) * LOG2E / np.sqrt(D)
        y = y.reshape(B * Hkv, G * w, n)
        rows = np.arange(G * w) % w
        vis = (key_offset + np.arange(n))[None, :] <= (p.N - w + rows)[:, None]
        return np.where(vis[None], y, -np.inf)

    def shard_stats(self, p, q, k_local, key_offset):
        y = self._logits(p, q, k_local, key_offset)
        m = y.max(axis=2)
        l = np.where(np.isfinite(m), np.exp2(y - np.where(np.isfinite(m), m, 0)[..., None]).sum(axis=2), 0.0)
        return torch.from_numpy(np.stack([m, l], axis=-1).astype(np.float32))

    def shard_scores(self, p, q, k_local, key_offset, ml_all):
        ml = ml_all.double().numpy()  # [W, U, nq, 2], merged in rank order
        M = ml[..., 0].max(axis=0)
        L = np.zeros_like(M)
        for w_ in range(ml.shape[0]):
            m_, l_ = ml[w_, ..., 0], ml[w_, ..., 1]
            L += np.where(np.isfinite(m_), l_ * np.exp2(np.where(np.isfinite(m_), m_ - M, 0)), 0.0)
        lse = M + np.log2(L)
        y = self._logits(p, q, k_local, key_offset)
        s = np.exp2(y - lse[..., None]).sum(axis=1)
        return torch.from_numpy(s.astype(np.float32).reshape(p.B, p.Hkv, -1))

    def pool(self, ext, lo, hi, kernel):
        from oracle import oracle as O
        x = ext.double().numpy()
        out = x.copy()
        out[:, :, lo:hi] = O.pool(x, lo, hi, kernel)[:, :, lo:hi]
        return torch.from_numpy(out.astype(np.float32))

    def hist(self, pooled, lo, hi, prefix, prefix_bits, digit_bits):
        x = pooled.numpy().reshape(-1, pooled.shape[-1])[:, lo:hi]
        keys = order_key(x)
        pre = prefix.numpy().view(np.uint32)
        nb = 1 << digit_bits
        out = np.zeros((x.shape[0], nb), dtype=np.int32)
        for r in range(x.shape[0]):
            kk = keys[r]
            if prefix_bits:
                kk = kk[(kk >> np.uint32(32 - prefix_bits)) == (pre[r] >> np.uint32(32 - prefix_bits))]
            d = (kk >> np.uint32(32 - prefix_bits - digit_bits)) & np.uint32(nb - 1)
            out[r] = np.bincount(d.astype(np.int64), minlength=nb)
        return torch.from_numpy(out)

    def pick(self, hist, hist_local, prefix_bits, need, prefix):
        """Per row, the bucket b (scanned from the top) holding the need-th largest key, the
        keys still needed inside it, the prefix extended by b, this rank's count in b."""
        h = hist.numpy().astype(np.int64)
        nb = h.shape[1]
        digit_bits = nb.bit_length() - 1
        need_in = need.numpy().astype(np.int64)
        from_top = np.cumsum(h[:, ::-1], axis=1)
        i = np.argmax(from_top >= need_in[:, None], axis=1)
        b = nb - 1 - i
        r = np.arange(h.shape[0])
        above = from_top[r, i] - h[r, b]
        pre = prefix.numpy().view(np.uint32) | (b.astype(np.uint32) << np.uint32(32 - prefix_bits - digit_bits))
        eq = hist_local.numpy()[r, b]
        return (torch.from_numpy((need_in - above).astype(np.int32)), torch.from_numpy(pre.view(np.int32).copy()),
                torch.from_numpy(eq.astype(np.int32)))

    def ties(self, eq_all, rank, need):
        e = eq_all.numpy().astype(np.int64)
        before = e[:rank].sum(axis=0) if rank > 0 else np.zeros(e.shape[1], dtype=np.int64)
        return torch.from_numpy(np.clip(need.numpy() - before, 0, e[rank]).astype(np.int32))

    def kept(self, sel, cnt, p, key_offset, n_local, cap):
        rows = sel.shape[0]
        pos = np.full((rows, cap), -1, dtype=np.int32)
        count = np.zeros(rows, dtype=np.int32)
        sinks = [t for t in range(p.n_sink) if key_offset <= t < key_offset + n_local]
        window = [t for t in range(p.N - p.window, p.N) if key_offset <= t < key_offset + n_local]
        for r in range(rows):
            kept = sinks + list(sel.numpy()[r, :int(cnt[r])]) + window
            pos[r, :len(kept)] = kept
            count[r] = len(kept)
        local = np.where(pos >= 0, pos - key_offset, 0).astype(np.int32)
        return torch.from_numpy(pos), torch.from_numpy(local), torch.from_numpy(count)

    def emit(self, pooled, lo, hi, thr, ties, pos_offset, cap):
        x = pooled.numpy().reshape(-1, pooled.shape[-1])
        T = thr.numpy().view(np.uint32)
        take = ties.numpy()
        out = np.zeros((x.shape[0], max(cap, 1)), dtype=np.int32)
        cnt = np.zeros(x.shape[0], dtype=np.int32)
        for r in range(x.shape[0]):
            keys = order_key(x[r, lo:hi])
            eq_rank = np.cumsum(keys == T[r]) - 1
            sel = (keys > T[r]) | ((keys == T[r]) & (eq_rank < take[r]))
            pos = pos_offset + lo + np.nonzero(sel)[0]
            out[r, :pos.size] = pos
            cnt[r] = pos.size
        return torch.from_numpy(out), torch.from_numpy(cnt)

    def gather(self, src, idx):
        B, H = src.shape[:2]
        return torch.stack([torch.stack([src[b, h, idx[b, h].long()] for h in range(H)]) for b in range(B)])


def _case():
    from long_context_kv_kvc_b200 import synth
    wl = synth.scaled(synth.LLAMA8B_32K, B=1, Hq=8, Hkv=2, N=700, window=32, kv_budget=150, n_hubs=12)
    inp = synth.make_inputs(wl, with_hidden=False)
    p = SimpleNamespace(B=wl.B, Hq=wl.Hq, Hkv=wl.Hkv, N=wl.N, window=wl.window, n_sink=wl.n_sink,
                        pool_kernel=wl.pool_kernel, kv_budget=wl.kv_budget)
    return wl, p, inp


def _worker(rank, world, port, cuts, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from long_context_kv_kvc_b200.sharded import TorchComm, sharded_compress
    wl, p, inp = _case()
    q = inp["q"][0]
    k, v = inp["k"][0], inp["v"]
    lo, hi = cuts[rank], cuts[rank + 1]
    res = sharded_compress(TorchComm(), NumpyOps(), p, q, k[:, :, lo:hi].contiguous(), v[:, :, lo:hi].contiguous(), lo)
    np.save(os.path.join(out_dir, f"pos{rank}.npy"), res["pos"].numpy())
    np.save(os.path.join(out_dir, f"count{rank}.npy"), res["count"].numpy())
    torch.save({"k": res["k"], "v": res["v"]}, os.path.join(out_dir, f"rows{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 350, 700], [0, 230, 455, 700], [0, 3, 680, 700]],
                         ids=["2-even", "3-uneven", "3-window-split"])
def test_sharded_selection_on_gloo_ranks(tmp_path, cuts):
    sys.path.insert(0, ROOT)
    world = len(cuts) - 1
    mp.start_processes(_worker, args=(world, _free_port(), cuts, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    from oracle import oracle as O
    from parity_util import check_index_sets
    wl, p, inp = _case()
    ref_pooled = O.pool(O.score(inp["q"], inp["k"], window=wl.window), wl.n_sink, wl.N - wl.window, wl.pool_kernel)
    kept = [[] for _ in range(wl.B * wl.Hkv)]
    for r in range(world):
        pos = np.load(tmp_path / f"pos{r}.npy").reshape(wl.B * wl.Hkv, -1)
        cnt = np.load(tmp_path / f"count{r}.npy").reshape(-1)
        rows = torch.load(tmp_path / f"rows{r}.pt")
        for i in range(wl.B * wl.Hkv):
            kept[i].extend(pos[i, :cnt[i]].tolist())
            b, h = divmod(i, wl.Hkv)
            src = inp["k"][0][b, h, torch.from_numpy(pos[i, :cnt[i]])]
            assert torch.equal(rows["k"][b, h, :cnt[i]], src)
            assert torch.equal(rows["v"][b, h, :cnt[i]], inp["v"][b, h, torch.from_numpy(pos[i, :cnt[i]])])
    idx = np.array(kept, dtype=np.int64).reshape(wl.B, wl.Hkv, -1)
    assert idx.shape[-1] == wl.kv_budget and np.all(np.diff(idx, axis=-1) > 0)
    # the band rule, and on this seeded case the very set of the unsharded oracle: the cut
    # into blocks changes nothing
    assert check_index_sets(idx, ref_pooled, wl.N, wl.n_sink, wl.window, wl.kv_budget) == 1.0
