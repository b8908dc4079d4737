"""Seeded synthetic inputs for attention-saliency KV-cache compaction.

This module only draws inputs.  It holds none of the compaction arithmetic (no scores,
softmax, pooling, selection or gather); both the CUDA path and the fp64 oracle consume
what it produces.

The pages evaluate on LLaMA-3.1-8B-class models (32 query heads, 8 KV heads, head
dimension 128) with contexts up to 128K on LongBench, RULER and needle-in-a-haystack
(FastKV page, sec. 4 "Ergebnisse"; StructKV page, "Belangrijkste Resultaten").  Neither
the weights nor the datasets are available, so the workloads below reproduce the shapes
with random data:

* q, K, V ~ N(0, 1) drawn in fp32;
* RoPE (rotate-half pairing d <-> d + D/2, theta = 500000, no frequency rescaling) applied
  to K at positions 0..N-1 and to the window queries at positions N-w..N-1;
* planted heavy hitters ("hubs"): per KV head, distinct positions drawn uniformly from the
  candidate range [S, N - w); their (rotated) K rows are overwritten with
  4 * mean(window queries of the head group) + N(0, 1) noise, so that they attract
  attention at any distance;
* the result is rounded to the workload dtype (bf16 round-to-nearest-even, or fp32).

Every block (sequence seed, layer, tensor kind, head) has its own PCG64 stream keyed by
numpy's SeedSequence, so blocks can be drawn in parallel threads and the values do not
depend on the thread count.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

# stream kinds
_Q, _K, _V, _HUB_POS, _HUB_NOISE, _HIDDEN, _SHARED_HUB_POS = 1, 2, 3, 4, 5, 6, 7

SCOPE_PER_KV_HEAD = 0
SCOPE_ALL_HEADS = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    window: int
    dtype: str  # "f32" | "bf16"
    pool_kernel: int
    kv_budget: int
    n_sink: int = 1
    n_layers: int = 1
    scope: int = SCOPE_PER_KV_HEAD
    tsp_rate: float = 0.0
    hidden_dim: int = 0
    rope: bool = True
    n_hubs: int = 256
    hub_shared_frac: float = 0.0  # fraction of hub positions shared across layers
    plant_sink: bool = False  # also plant key 0 as a heavy key
    seeds: tuple = (0,)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The workloads, by what they are.
TINY = Workload("tiny-gqa4-2k-f32", B=1, Hq=4, Hkv=1, N=2048, D=128, window=8, dtype="f32",
                pool_kernel=7, kv_budget=256, n_sink=1, rope=False, n_hubs=32, plant_sink=True)
LLAMA8B_32K = Workload("llama8b-32k", B=1, Hq=32, Hkv=8, N=32768, D=128, window=32, dtype="bf16",
                       pool_kernel=7, kv_budget=2048)
LLAMA8B_128K_B4 = Workload("llama8b-128k-b4", B=4, Hq=32, Hkv=8, N=131072, D=128, window=32,
                           dtype="bf16", pool_kernel=7, kv_budget=4096, seeds=(0, 1, 2, 3))
LLAMA8B_128K_B1 = Workload("llama8b-128k-b1", B=1, Hq=32, Hkv=8, N=131072, D=128, window=32,
                           dtype="bf16", pool_kernel=7, kv_budget=4096)
STRUCTKV_8L_32K = Workload("structkv-8layer-32k", B=1, Hq=32, Hkv=8, N=32768, D=128, window=32,
                           dtype="bf16", pool_kernel=7, kv_budget=2048, n_layers=8,
                           scope=SCOPE_ALL_HEADS, hub_shared_frac=0.6)
FASTKV_TSP_64K = Workload("fastkv-tsp20-64k", B=1, Hq=32, Hkv=8, N=65536, D=128, window=32,
                          dtype="bf16", pool_kernel=7, kv_budget=1024, tsp_rate=0.2, hidden_dim=4096)

WORKLOADS = {w.name: w for w in (TINY, LLAMA8B_32K, LLAMA8B_128K_B4, LLAMA8B_128K_B1, STRUCTKV_8L_32K,
                                 FASTKV_TSP_64K)}


def _stream(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, key)])))


def _normal(seed: int, key: tuple, shape) -> np.ndarray:
    return _stream(seed, *key).standard_normal(size=shape, dtype=np.float32)


def _rope_tables(positions: np.ndarray, D: int, theta: float):
    inv_freq = theta ** (-np.arange(0, D // 2, dtype=np.float64) * 2.0 / D)
    ang = positions.astype(np.float64)[:, None] * inv_freq[None, :]
    return torch.from_numpy(np.cos(ang).astype(np.float32)), torch.from_numpy(np.sin(ang).astype(np.float32))


def _apply_rope(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    """x [..., P, D] fp32; rotate-half pairing of d and d + D/2."""
    h = x.shape[-1] // 2
    a, b = x[..., :h], x[..., h:]
    return torch.cat((a * cos - b * sin, a * sin + b * cos), dim=-1)


def hub_positions(wl: Workload, seed: int, layer: int, head: int) -> np.ndarray:
    """Distinct planted positions in [S, N - w) for one (sequence, layer, KV head)."""
    lo, hi = wl.n_sink, wl.N - wl.window
    n_c = hi - lo
    n = min(wl.n_hubs, n_c)
    n_shared = int(round(wl.hub_shared_frac * n)) if wl.n_layers > 1 else 0
    shared = np.sort(_stream(seed, _SHARED_HUB_POS, head).permutation(n_c)[:n_shared])
    rest_pool = np.setdiff1d(np.arange(n_c), shared, assume_unique=True)
    own = _stream(seed, layer, _HUB_POS, head).permutation(rest_pool.size)[: n - n_shared]
    return np.sort(np.concatenate([shared, rest_pool[own]])) + lo


def make_inputs(wl: Workload, seeds=None, threads: int = 8, with_v: bool = True,
                with_hidden: bool = True) -> dict:
    """Draw one batch of the workload on the CPU.

    Returns a dict of CPU tensors in the workload dtype:
      q      [L, B, Hq, w, D]   window queries (post-RoPE)
      k      [L, B, Hkv, N, D]  keys (post-RoPE, hubs planted)
      v      [B, Hkv, N, D]     values of the last layer (the one that is compacted)
      hidden [B, N, hidden_dim] hidden-state rows (only when tsp_rate > 0)
      hubs   {(layer, b, head): positions}
    Sequence b uses seed ``seeds[b]`` (default: the workload's seeds).
    """
    seeds = tuple(wl.seeds if seeds is None else seeds)
    if len(seeds) != wl.B:
        raise ValueError(f"need {wl.B} seeds, got {len(seeds)}")
    L, B, Hq, Hkv, N, D, w = wl.n_layers, wl.B, wl.Hq, wl.Hkv, wl.N, wl.D, wl.window
    G = wl.G
    q = torch.empty((L, B, Hq, w, D), dtype=torch.float32)
    k = torch.empty((L, B, Hkv, N, D), dtype=torch.float32)
    v = torch.empty((B, Hkv, N, D), dtype=torch.float32) if with_v else None
    hidden = None
    if with_hidden and wl.tsp_rate > 0 and wl.hidden_dim > 0:
        hidden = torch.empty((B, N, wl.hidden_dim), dtype=torch.float32)

    jobs = []
    for layer in range(L):
        for b in range(B):
            for g in range(Hq):
                jobs.append((q, (layer, b, g), seeds[b], (layer, _Q, g), (w, D)))
            for h in range(Hkv):
                jobs.append((k, (layer, b, h), seeds[b], (layer, _K, h), (N, D)))
    if v is not None:
        for b in range(B):
            for h in range(Hkv):
                jobs.append((v, (b, h), seeds[b], (L - 1, _V, h), (N, D)))
    if hidden is not None:
        for b in range(B):
            jobs.append((hidden, (b,), seeds[b], (0, _HIDDEN, 0), (N, wl.hidden_dim)))

    def run(job):
        dst, index, seed, key, shape = job
        dst[index].copy_(torch.from_numpy(_normal(seed, key, shape)))

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(run, jobs))

    if wl.rope:
        theta = 500000.0
        cos_k, sin_k = _rope_tables(np.arange(N), D, theta)
        cos_q, sin_q = _rope_tables(np.arange(N - w, N), D, theta)
        q = _apply_rope(q, cos_q, sin_q)
        for layer in range(L):
            for b in range(B):
                k[layer, b] = _apply_rope(k[layer, b], cos_k, sin_k)

    hubs = {}
    for layer in range(L):
        for b in range(B):
            for h in range(Hkv):
                pos = hub_positions(wl, seeds[b], layer, h)
                if wl.plant_sink:
                    pos = np.concatenate([[0], pos])
                mean_q = q[layer, b, h * G:(h + 1) * G].reshape(-1, D).mean(dim=0)
                noise = torch.from_numpy(_normal(seeds[b], (layer, _HUB_NOISE, h), (pos.size, D)))
                k[layer, b, h, torch.from_numpy(pos)] = 4.0 * mean_q + noise
                hubs[(layer, b, h)] = pos

    td = wl.torch_dtype
    out = {"q": q.to(td).contiguous(), "k": k.to(td).contiguous(), "hubs": hubs}
    out["v"] = v.to(td).contiguous() if v is not None else None
    out["hidden"] = hidden.to(td).contiguous() if hidden is not None else None
    return out


def scaled(wl: Workload, **kw) -> Workload:
    """A smaller copy of a workload (same structure), e.g. for parity tests."""
    w = wl.replace(**kw)
    if "seeds" not in kw and len(w.seeds) != w.B:
        w = w.replace(seeds=tuple(range(w.B)))
    return w
