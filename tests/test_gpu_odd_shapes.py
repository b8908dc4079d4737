"""An odd-shape sweep of the compaction, Chunked Soft Matching and sequence sharding through
the C ABI, against the fp64 oracle.

Shapes: N one past a 128-key tile, below one tile, and not a multiple of it; windows of 1
to 128 rows (G * window up to 256); no sinks to several; pool widths 1 to 13; budgets at
both ends of their range (n_sink + window + 1 and N) and between; every path (tensor cores,
CUDA cores, fp32).  The same module runs once more against the range-checking library
(libkvc_checks.so, see test_gpu_checks.py), where every case must also leave the device
error word clear.
"""
import numpy as np
import pytest
import torch

from long_context_kv_kvc_b200 import synth
from oracle import oracle as O
from parity_util import check_csm_row, check_index_sets, run_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_kv_kvc_b200 import build, kvc
    if not kvc.CHECKS:
        build.build()
    torch.cuda.set_device(0)
    return kvc


# (Hq, Hkv, N, window, n_sink, pool_kernel, budget); budget None = n_sink + window + 1
SHAPES = [
    (4, 1, 129, 1, 0, 1, None),       # one key past a tile, the smallest window and budget
    (4, 1, 129, 7, 5, 13, 129),       # budget = N
    (8, 2, 255, 33, 1, 3, None),      # window 33: G * w = 132 query rows (two row blocks)
    (8, 2, 257, 32, 1, 7, 257),
    (8, 1, 1153, 32, 4, 7, 600),      # G * w = 256, the most query rows a unit has
    (4, 4, 1000, 64, 2, 5, None),     # G = 1
    (8, 2, 4097, 17, 3, 9, 1000),
    (4, 1, 31, 5, 2, 3, 8),           # shorter than one tile
    (2, 2, 130, 128, 1, 1, 130),      # window of 128 rows, budget = N
    (4, 2, 385, 3, 0, 11, 200),       # no sinks, a wide pool
]


def _wl(shape, dtype="bf16", **kw):
    Hq, Hkv, N, w, S, P, budget = shape
    budget = S + w + 1 if budget is None else budget
    base = synth.LLAMA8B_32K if dtype == "bf16" else synth.TINY
    return synth.scaled(base, B=1, Hq=Hq, Hkv=Hkv, N=N, window=w, n_sink=S, pool_kernel=P, kv_budget=budget,
                        n_hubs=max(1, min(8, (N - S - w) // 4)), **kw)


@pytest.mark.parametrize("flags", [0, 1], ids=["tensor_cores", "cuda_cores"])
@pytest.mark.parametrize("shape", range(len(SHAPES)))
def test_compress_odd_shapes_bf16(K, shape, flags):
    run_case(K, _wl(SHAPES[shape]), flags=flags)


@pytest.mark.parametrize("shape", [0, 2, 5, 7])
def test_compress_odd_shapes_f32(K, shape):
    run_case(K, _wl(SHAPES[shape], dtype="f32"))


def test_compress_odd_layers_all_heads_and_tsp(K):
    wl = synth.scaled(synth.STRUCTKV_8L_32K, N=999, n_layers=2, window=16, n_sink=1, pool_kernel=7, kv_budget=18,
                      n_hubs=8)
    run_case(K, wl)
    wl = synth.scaled(synth.FASTKV_TSP_64K, N=777, window=9, n_sink=3, pool_kernel=5, kv_budget=300,
                      hidden_dim=256, n_hubs=8)
    run_case(K, wl)


def test_topk_long_row_single_cta_path(K):
    """Rows whose candidates do not fit the 8-CTA clusters' shared memory take the one-CTA
    radix select; pool then select at that length, budgets at both ends."""
    g = np.random.default_rng(5)
    N = 200_003
    raw = np.round(g.random((1, 2, N)), 4).astype(np.float32)
    for S, w, P, budget in [(1, 7, 5, 9), (0, 1, 1, N), (3, 31, 3, 4099)]:
        pooled = torch.empty((1, 2, N), dtype=torch.float32, device="cuda")
        K.kvc_pool(torch.from_numpy(raw).cuda(), pooled, S, N - w, P)
        idx = torch.empty((1, 2, budget), dtype=torch.int32, device="cuda")
        K.kvc_topk(pooled, S, w, budget, idx)
        assert K.kvc_poll_error() == K.KVC_OK
        ref = O.select(O.pool(raw.astype(np.float64), S, N - w, P), S, w, budget)
        assert np.array_equal(idx.cpu().numpy(), ref), (S, w, P, budget)


# (N, n_sink, window, chunk, ratio, dtype)
CSM_SHAPES = [
    (131, 0, 1, 2, 0.5, torch.bfloat16),
    (259, 3, 0, 128, 0.5, torch.bfloat16),
    (333, 1, 5, 6, 0.4, torch.float32),
    (1001, 7, 33, 126, 0.2, torch.bfloat16),
    (129, 64, 64, 16, 0.5, torch.bfloat16),  # one candidate: nothing to merge
]


@pytest.mark.parametrize("shape", range(len(CSM_SHAPES)))
def test_csm_odd_shapes(K, shape):
    N, S, w, chunk, ratio, dtype = CSM_SHAPES[shape]
    g = torch.Generator().manual_seed(200 + shape)
    k = torch.randn(1, 2, N, 128, generator=g)
    k[:, :, 1::7] = 1.25 * k[:, :, 0:-1:7][:, :, : k[:, :, 1::7].shape[2]]  # near-duplicate neighbours
    k, v = k.to(dtype), torch.randn(1, 2, N, 128, generator=g).to(dtype)
    deg = torch.randint(1, 5, (1, 2, N), generator=g, dtype=torch.int32)
    out = K.kvc_csm(k.cuda(), v.cuda(), S, w, chunk, ratio, deg=deg.cuda())
    assert K.kvc_poll_error() == K.KVC_OK
    for h in range(2):
        check_csm_row(k[0, h], v[0, h], deg[0, h].numpy(), out["k_out"][0, h].cpu(), out["v_out"][0, h].cpu(),
                      out["deg_out"][0, h].cpu().numpy(), out["pos_out"][0, h].cpu().numpy(), S, w, chunk, ratio,
                      dtype)


@pytest.mark.parametrize("cuts", [(0, 129, 300, 513), (0, 1, 512, 513), (0, 256, 257, 513)],
                         ids=["ragged", "one_key_block", "one_key_middle"])
def test_sharded_compress_odd_cuts(K, cuts):
    """Sequence sharding over blocks of 1 to 512 keys (the ranks are host threads on one GPU);
    a block must hold the pool's half-width (pool_kernel - 1) / 2 of keys, here 1."""
    from long_context_kv_kvc_b200.sharded import GpuOps, sharded_compress
    from test_gpu_sharded import run_ranks
    wl = synth.scaled(synth.LLAMA8B_32K, B=1, Hq=8, Hkv=2, N=513, window=9, n_sink=2, pool_kernel=3, kv_budget=40,
                      n_hubs=8)
    inp = synth.make_inputs(wl, with_hidden=False)
    q, k, v = inp["q"][0].cuda(), inp["k"][0].cuda(), inp["v"].cuda()
    p = K.params_for(wl)
    K.kvc_poll_error()
    torch.cuda.synchronize()

    def rank_fn(comm, a, b):
        return sharded_compress(comm, GpuOps(), p, q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(), a)

    res = run_ranks(list(cuts), rank_fn)
    torch.cuda.synchronize()
    assert K.kvc_poll_error() == K.KVC_OK
    rows = wl.B * wl.Hkv
    kept = [[] for _ in range(rows)]
    for out in res:
        pos = out["pos"].cpu().numpy().reshape(rows, -1)
        cnt = out["count"].cpu().numpy().reshape(-1)
        for i in range(rows):
            kept[i].extend(pos[i, :cnt[i]].tolist())
    idx = np.array(kept, dtype=np.int64).reshape(wl.B, wl.Hkv, -1)
    ref_pooled = O.pool(O.score(inp["q"], inp["k"], window=wl.window), wl.n_sink, wl.N - wl.window, wl.pool_kernel)
    check_index_sets(idx, ref_pooled, wl.N, wl.n_sink, wl.window, wl.kv_budget)
