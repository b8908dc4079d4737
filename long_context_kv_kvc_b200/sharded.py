"""Sequence-sharded compaction: one GPU per contiguous block of the sequence.

For contexts whose keys do not fit one GPU, rank r holds keys [off_r, off_r + n_r) of every
(batch, KV head) and all window queries.  The pages describe single-device scoring; the
sharded variant computes the same definition (window softmax -> per-KV-head sum -> max-pool
over the candidates -> top-k_sel plus sinks and window, ties to the lower position) with one
small exchange per step, all of a few KiB:

  1. every rank's (max, sum) of each window row over its keys, all-gathered; each rank
     merges them in rank order into the same log-sum-exp and scores its keys;
  2. a halo of (P - 1) / 2 scores from each neighbour for the pool at the block edges;
  3. a radix select over the candidates of all ranks: per digit (11, 11, 10 bits) each
     rank's histogram of the candidates matching the prefix so far, summed over ranks;
  4. every rank's number of candidates equal to the threshold, all-gathered: rank r takes
     the ties left after the lower ranks' (ties go to the lower positions);
  5. each rank gathers its kept rows; the compact cache is the ranks' parts in rank order.

Every step on the data runs in the library's kernels (`Ops`), the radix bucket picks, the
split of ties and the kept positions included, so the data stays on the device and the host
does not wait for it; this module holds the order of the steps and the exchanges (`Comm`),
both replaceable so that the host logic can be exercised with CPU ranks.
"""
from __future__ import annotations

import torch

DIGITS = (11, 11, 10)


class TorchComm:
    """Collectives of torch.distributed (NCCL between GPUs, gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        parts = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts)

    def all_reduce_sum(self, t: torch.Tensor) -> torch.Tensor:
        t = t.clone()
        self.dist.all_reduce(t, group=self.group)
        return t


class GpuOps:
    """The steps on the data, as the library's kernels."""

    def __init__(self):
        from . import kvc
        self.kvc = kvc
        self._ws = None

    def _workspace(self, p, n_local, device):
        need = self.kvc.kvc_shard_workspace_size(p, n_local)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
        return self._ws

    def shard_stats(self, p, q, k_local, key_offset):
        U, nq = p.B * p.Hkv, p.Hq // p.Hkv * p.window
        ml = torch.empty((U, nq, 2), dtype=torch.float32, device=k_local.device)
        self.kvc.kvc_shard_stats(p, q, k_local, key_offset, ml, self._workspace(p, k_local.shape[-2], k_local.device))
        return ml

    def shard_scores(self, p, q, k_local, key_offset, ml_all):
        n_local = k_local.shape[-2]
        scores = torch.empty((p.B, p.Hkv, n_local), dtype=torch.float32, device=k_local.device)
        self.kvc.kvc_shard_scores(p, q, k_local, key_offset, ml_all.contiguous(), scores,
                                  self._workspace(p, n_local, k_local.device))
        return scores

    def pool(self, ext, lo, hi, kernel):
        out = torch.empty_like(ext)
        B, H, n = ext.shape
        self.kvc.kvc_pool(ext, out, lo, hi, kernel)
        return out

    def hist(self, pooled, lo, hi, prefix, prefix_bits, digit_bits):
        rows = pooled.shape[0] * pooled.shape[1]
        hist = torch.empty((rows, 1 << digit_bits), dtype=torch.int32, device=pooled.device)
        self.kvc.kvc_select_hist(pooled, lo, hi, prefix.to(pooled.device), prefix_bits, digit_bits, hist)
        return hist

    def pick(self, hist, hist_local, prefix_bits, need, prefix):
        """One digit: the bucket of every row's need-th largest key (device); returns the
        updated need and prefix and this rank's count in the bucket."""
        need, prefix = need.clone(), prefix.clone()
        eq_local = torch.empty_like(need)
        # a collective may hand back the summed counts widened to int64
        self.kvc.kvc_select_pick(hist.to(torch.int32).contiguous(), hist_local, prefix_bits, need, prefix, eq_local)
        return need, prefix, eq_local

    def ties(self, eq_all, rank, need):
        take = torch.empty_like(need)
        self.kvc.kvc_select_ties(eq_all.to(torch.int32).contiguous(), rank, need, take)
        return take

    def kept(self, sel, cnt, p, key_offset, n_local, cap):
        rows = sel.shape[0]
        pos = torch.empty((rows, cap), dtype=torch.int32, device=sel.device)
        local = torch.empty_like(pos)
        count = torch.empty((rows,), dtype=torch.int32, device=sel.device)
        self.kvc.kvc_select_kept(sel, cnt, p.N, p.n_sink, p.window, key_offset, n_local, pos, local, count)
        return pos, local, count

    def emit(self, pooled, lo, hi, thr, ties, pos_offset, cap):
        rows = pooled.shape[0] * pooled.shape[1]
        out = torch.empty((rows, max(cap, 1)), dtype=torch.int32, device=pooled.device)
        count = torch.empty((rows,), dtype=torch.int32, device=pooled.device)
        self.kvc.kvc_select_emit(pooled, lo, hi, thr.to(pooled.device), ties.to(pooled.device), pos_offset, out, count)
        return out, count

    def gather(self, src, idx):
        B, H, _, D = src.shape
        dst = torch.empty((B, H, idx.shape[-1], D), dtype=src.dtype, device=src.device)
        self.kvc.kvc_gather(src, idx, dst)
        return dst


def sharded_compress(comm, ops, p, q, k_local, v_local, key_offset: int):
    """One rank's part of the sharded compaction.

    p         kvc Params of the whole sequence (N = all keys; n_layers 1, per-KV-head scope)
    q         [B, Hq, window, D] window queries (the same on every rank)
    k_local, v_local  [B, Hkv, n_local, D]: keys key_offset .. key_offset + n_local - 1
    Returns {"pos": [B, Hkv, cap] int32 global positions this rank keeps (ascending, padded
    with -1), "count": [B, Hkv] int32 kept per row, "k", "v": the kept rows [B, Hkv, cap, D]
    (rows past count are padding), "scores": this rank's scores [B, Hkv, n_local]}, all on the
    ranks' device; cap = min(n_local, kv_budget).
    """
    B, H, n_local, D = k_local.shape
    N, S, w, P = p.N, p.n_sink, p.window, p.pool_kernel
    rows = B * H
    dev = k_local.device
    k_sel = p.kv_budget - S - w
    h = (P - 1) // 2
    if n_local < max(h, 1):
        raise ValueError("every block must hold at least (pool_kernel - 1) / 2 keys")

    # 1. softmax normalisers over all ranks, then this block's scores
    ml = ops.shard_stats(p, q, k_local, key_offset)
    ml_all = comm.all_gather(ml)
    scores = ops.shard_scores(p, q, k_local, key_offset, ml_all)

    # 2. pool with the neighbours' edge scores (positions outside C are never pooled)
    n_ext = n_local + 2 * h
    ext = torch.zeros((B, H, n_ext), dtype=torch.float32, device=dev)
    ext[:, :, h:h + n_local] = scores
    if h > 0:
        edges = torch.cat([scores[:, :, :h], scores[:, :, n_local - h:]], dim=2).contiguous()
        all_edges = comm.all_gather(edges)
        if comm.rank > 0:
            ext[:, :, :h] = all_edges[comm.rank - 1][:, :, h:]
        if comm.rank < comm.world - 1:
            ext[:, :, n_local + h:] = all_edges[comm.rank + 1][:, :, :h]
    base = key_offset - h                                      # global position of ext[0]
    c_lo, c_hi = max(S, base), min(N - w, base + n_ext)        # candidates C inside ext
    lo, hi = c_lo - base, max(c_hi - base, c_lo - base)
    pooled = ops.pool(ext, lo, hi, P) if hi > lo else ext
    # this block's own candidates, in ext coordinates
    own_lo, own_hi = max(S, key_offset) - base, min(N - w, key_offset + n_local) - base
    own_hi = max(own_hi, own_lo)

    # 3. radix select over every rank's candidates: per digit, the histograms summed over
    #    ranks, then every rank picks the same bucket (on the device)
    need = torch.full((rows,), k_sel, dtype=torch.int32, device=dev)
    prefix = torch.zeros((rows,), dtype=torch.int32, device=dev)
    bits = 0
    eq_local = None
    for d in DIGITS:
        hist_local = ops.hist(pooled, own_lo, own_hi, prefix, bits, d)
        hist = comm.all_reduce_sum(hist_local)
        need, prefix, eq_local = ops.pick(hist, hist_local, bits, need, prefix)
        bits += d

    # 4. ties: the lower ranks take theirs first
    eq_all = comm.all_gather(eq_local)
    take = ops.ties(eq_all, comm.rank, need)
    cap_sel = max(own_hi - own_lo, 1)
    sel, cnt = ops.emit(pooled, own_lo, own_hi, prefix, take, base, cap_sel)

    # 5. kept positions of this block: sinks, the selection, the window; then the rows
    cap = max(1, min(n_local, p.kv_budget))
    pos, local, count = ops.kept(sel, cnt, p, key_offset, n_local, cap)
    idx = local.reshape(B, H, cap)
    return {"pos": pos.reshape(B, H, cap), "count": count.reshape(B, H), "k": ops.gather(k_local, idx),
            "v": ops.gather(v_local, idx), "scores": scores}
