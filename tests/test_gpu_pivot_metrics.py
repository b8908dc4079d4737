"""Parity of the pivot-detection metrics through the C ABI with the fp64 oracle.

Window-row attention entropy (kvc_score_entropy, taken in the scoring pass) and the kept
mass / candidate variance of score rows (kvc_row_stats), on seeded inputs of several
shapes, both scoring paths, and sampled rows of the full 128K x 4 workload.

Entropy tolerance: the GPU forms H = ln2 (log2 L - T / L) from fp32 sums of 2^(y - ref)
and 2^(y - ref) (y - ref) (special-function-unit exp2, relative error ~2^-22 per term)
gathered in fp64; with |y - ref| below ~40 that bounds the error near 1e-5 nats, so the
test allows |dH| <= 1e-3 H + 1e-4.  Row statistics are fp64 sums of the same fp32 scores
the oracle reads, rounded once to fp32: relative 1e-6.
"""
import numpy as np
import pytest
import torch

from long_context_kv_kvc_b200 import synth
from oracle import oracle as O

pytestmark = pytest.mark.gpu

H_RTOL, H_ATOL = 1e-3, 1e-4


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_kv_kvc_b200 import build
    build.build()
    from long_context_kv_kvc_b200 import kvc
    torch.cuda.set_device(0)
    return kvc


def check_entropy(got, ref):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    bound = H_RTOL * np.abs(ref) + H_ATOL
    assert np.all(np.isfinite(got)), "non-finite entropy"
    assert np.all(err <= bound), f"{(err > bound).sum()} rows outside tolerance; worst {err.max():.3e}"
    return float(err.max())


ENTROPY_CASES = [
    synth.TINY,
    synth.scaled(synth.LLAMA8B_32K, B=1, Hq=8, Hkv=2, N=1000, kv_budget=200, n_hubs=16),
    synth.scaled(synth.LLAMA8B_32K, B=2, Hq=4, Hkv=1, N=4133, window=8, kv_budget=500, n_hubs=64),
    synth.scaled(synth.LLAMA8B_32K, B=1, Hq=32, Hkv=8, N=2053, kv_budget=1024, n_hubs=32),
    synth.scaled(synth.STRUCTKV_8L_32K, n_layers=3, N=1531, kv_budget=300, n_hubs=16),
]


@pytest.mark.parametrize("flags", [0, 1], ids=["default", "simt"])
@pytest.mark.parametrize("case", range(len(ENTROPY_CASES)))
def test_entropy_matches_oracle(K, case, flags):
    wl = ENTROPY_CASES[case]
    inp = synth.make_inputs(wl, with_v=False, with_hidden=False)
    q, k = inp["q"].cuda(), inp["k"].cuda()
    p = K.params_for(wl, flags=flags)
    ws = torch.empty(K.kvc_workspace_size(p), dtype=torch.uint8, device="cuda")
    Hs = wl.Hkv if wl.scope == K.KVC_SCOPE_PER_KV_HEAD else 1
    scores = torch.empty((wl.B, Hs, wl.N), dtype=torch.float32, device="cuda")
    ent = torch.full((wl.n_layers, wl.B, wl.Hq, wl.window), float("nan"), dtype=torch.float32, device="cuda")
    K.kvc_score_entropy(p, q, k, scores, ent, ws)
    assert K.kvc_poll_error() == K.KVC_OK
    check_entropy(ent.cpu().numpy(), O.entropy(inp["q"], inp["k"], window=wl.window))
    # the entropy pass gives the same scores as kvc_score, bit for bit
    plain = torch.empty_like(scores)
    K.kvc_score(p, q, k, plain, ws)
    assert torch.equal(plain, scores)


def test_entropy_full_size_128k_batch4_sampled(K):
    wl = synth.LLAMA8B_128K_B4
    inp = synth.make_inputs(wl, with_v=False, with_hidden=False)
    q, k = inp["q"].cuda(), inp["k"].cuda()
    p = K.params_for(wl)
    ws = torch.empty(K.kvc_workspace_size(p), dtype=torch.uint8, device="cuda")
    scores = torch.empty((wl.B, wl.Hkv, wl.N), dtype=torch.float32, device="cuda")
    ent = torch.empty((1, wl.B, wl.Hq, wl.window), dtype=torch.float32, device="cuda")
    K.kvc_score_entropy(p, q, k, scores, ent, ws)
    assert K.kvc_poll_error() == K.KVC_OK
    got = ent.cpu().numpy().reshape(-1)
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got <= np.log(wl.N) + 1e-4)
    rows = np.random.default_rng(11).choice(got.size, 48, replace=False).astype(np.int32)
    rows = np.concatenate([rows, [0, wl.window - 1, got.size - 1]]).astype(np.int32)
    check_entropy(got[rows], O.entropy(inp["q"], inp["k"], window=wl.window, rows=rows))


def test_row_stats_match_oracle(K):
    g = torch.Generator().manual_seed(12)
    B, H, N, S, w, budget = 3, 4, 70001, 1, 32, 4096
    scores = torch.rand((B, H, N), generator=g, dtype=torch.float32) ** 3
    scores[1, 2] = 0.25  # a constant row: variance 0
    dev = scores.cuda()
    idx = torch.empty((B, H, budget), dtype=torch.int32, device="cuda")
    K.kvc_topk(dev, S, w, budget, idx)
    km = torch.full((B, H), float("nan"), device="cuda")
    cv = torch.full((B, H), float("nan"), device="cuda")
    K.kvc_row_stats(dev, S, w, cv, idx=idx, kept_mass=km)
    assert K.kvc_poll_error() == K.KVC_OK
    ref_km, ref_cv = O.row_stats(scores.double().numpy(), S, w, idx.cpu().numpy())
    np.testing.assert_allclose(km.cpu().numpy(), ref_km, rtol=1e-6)
    np.testing.assert_allclose(cv.cpu().numpy(), ref_cv, rtol=1e-6, atol=1e-30)
    assert cv[1, 2].item() == 0.0
    # without indices only the variance is written
    km2 = torch.full((B, H), -1.0, device="cuda")
    cv2 = torch.empty((B, H), device="cuda")
    K.kvc_row_stats(dev, S, w, cv2, kept_mass=km2)
    assert torch.equal(cv2, cv) and torch.all(km2 == -1.0)


def test_row_stats_bad_index_and_arguments(K):
    dev = torch.ones((1, 1, 100), device="cuda")
    idx = torch.arange(10, dtype=torch.int32, device="cuda").view(1, 1, 10)
    idx[0, 0, 3] = 100  # out of range: left out and reported
    km = torch.empty((1, 1), device="cuda")
    cv = torch.empty((1, 1), device="cuda")
    K.kvc_row_stats(dev, 1, 8, cv, idx=idx, kept_mass=km)
    assert K.kvc_poll_error() == K.KVC_ERR_INDEX
    assert km.item() == pytest.approx(9 / 100, rel=1e-7)
    with pytest.raises(K.KvcError):
        K.kvc_row_stats(dev, 60, 40, cv)  # n_sink + window >= N
    assert K.kvc_poll_error() == K.KVC_OK
