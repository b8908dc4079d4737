"""Decode-side consumers of the clustered cache, through the C ABI, against the fp64 oracle.

* kvc_decode_attention: attention over centroids with ln(degree) in the logits (CentroidKV
  page, sec. 4); bf16 caches take the tensor-core kernel, fp32 caches the CUDA-core one.
  Tolerance: the GPU forms fp32 logits (|error| ~1e-6 in base-2 units),
  fp32 exponentials and fp32 sums over spans of a few thousand rows, merged in fp32; the
  resulting error is a small multiple of 2^-24 times sqrt(rows) relative to the weighted
  magnitude sum_t p_t |v_t|, so the test allows 5e-5 of that magnitude plus 1e-6.
* kvc_append and the strided form of kvc_csm (row capacity, carried positions).
* CentroidCache: a decode loop with a round after prefill and one every g steps (sec. 2),
  each round checked against the oracle on the GPU's own pre-round cache, every step's
  attention against the oracle on the GPU's cache.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity_util import check_csm_row as check_row

pytestmark = pytest.mark.gpu

RTOL_W = 5e-5


@pytest.fixture(scope="module")
def K():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_kv_kvc_b200 import build
    build.build()
    from long_context_kv_kvc_b200 import kvc
    torch.cuda.set_device(0)
    return kvc


def weighted_magnitude(q, k, v, deg):
    """sum_t p_t |v_t| in fp64 (the scale of the attention output's rounding error)."""
    B, Hq, nq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    qq = q.double().numpy()
    kk = k.double().numpy()
    vv = np.abs(v.double().numpy())
    out = np.empty((B, Hq, nq, D))
    for b in range(B):
        for g in range(Hq):
            h = g // G
            x = qq[b, g] @ kk[b, h].T / np.sqrt(D)
            if deg is not None:
                x = x + np.log(np.asarray(deg[b, h], dtype=np.float64))
            x -= x.max(axis=1, keepdims=True)
            p = np.exp(x)
            p /= p.sum(axis=1, keepdims=True)
            out[b, g] = p @ vv[b, h]
    return out


def check_attention(got, q, k, v, deg):
    ref = O.centroid_attention(q, k, v, None if deg is None else np.asarray(deg))
    scale = weighted_magnitude(q, k, v, deg)
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    bound = RTOL_W * scale + 1e-6
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), f"worst {(err / scale).max():.2e} of the weighted magnitude"


CASES = [  # B, Hq, Hkv, nq, n, ld, dtype, degrees
    (1, 4, 1, 1, 37, 37, torch.float32, False),
    (2, 32, 8, 1, 5000, 5003, torch.bfloat16, True),
    (1, 8, 2, 2, 777, 800, torch.bfloat16, True),   # 8 query rows per KV head
    (3, 6, 3, 1, 300, 300, torch.float32, True),    # 2 rows, padded to 4
    (1, 12, 4, 1, 257, 260, torch.bfloat16, False),  # 3 rows, padded to 4
    (1, 8, 1, 1, 1, 1, torch.bfloat16, True),       # a single cached row
    (1, 4, 4, 1, 4133, 4133, torch.float32, True),  # G = 1
    (1, 4, 1, 1, 20000, 20000, torch.bfloat16, True),  # one unit over every CTA's range
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_decode_attention_matches_oracle(K, case):
    B, Hq, Hkv, nq, n, ld, dtype, with_deg = CASES[case]
    g = torch.Generator().manual_seed(100 + case)
    q = torch.randn(B, Hq, nq, 128, generator=g).to(dtype)
    k = torch.randn(B, Hkv, ld, 128, generator=g).to(dtype)
    v = torch.randn(B, Hkv, ld, 128, generator=g).to(dtype)
    deg = torch.randint(1, 9, (B, Hkv, ld), generator=g, dtype=torch.int32) if with_deg else None
    out = K.kvc_decode_attention(q.cuda(), k.cuda(), v.cuda(), deg=None if deg is None else deg.cuda(), n=n)
    assert K.kvc_poll_error() == K.KVC_OK
    check_attention(out.cpu().numpy(), q, k[:, :, :n], v[:, :, :n], None if deg is None else deg[:, :, :n].numpy())


def test_decode_degree_equals_replication_on_gpu(K):
    # a row of degree n attends like n copies of itself (exact in arithmetic; fp32 here)
    g = torch.Generator().manual_seed(7)
    Hq, Hkv, n = 8, 2, 900
    q = torch.randn(1, Hq, 1, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(1, Hkv, n, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(1, Hkv, n, 128, generator=g).to(torch.bfloat16)
    deg = torch.randint(1, 4, (1, Hkv, n), generator=g, dtype=torch.int32)
    a = K.kvc_decode_attention(q.cuda(), k.cuda(), v.cuda(), deg=deg.cuda()).cpu()
    for h in range(Hkv):
        reps = deg[0, h].long()
        kr = k[:, h:h + 1, :].repeat_interleave(reps, dim=2)
        vr = v[:, h:h + 1, :].repeat_interleave(reps, dim=2)
        b = K.kvc_decode_attention(q[:, 4 * h:4 * h + 4].cuda(), kr.cuda(), vr.cuda()).cpu()
        scale = weighted_magnitude(q[:, 4 * h:4 * h + 4], kr, vr, None)
        assert np.all(np.abs((a[:, 4 * h:4 * h + 4] - b).numpy()) <= 2 * RTOL_W * scale + 1e-6)


def test_decode_attention_full_size_128k_batch4(K):
    """After one clustering round of the 128K x 4 cache (bf16, 8 KV heads, r = 0.25, chunks
    of 64: 98313 centroids), 32 query heads attend; four (batch, KV head) units are checked
    against the oracle and every output for finiteness and the convex-hull bound."""
    B, Hq, Hkv, N = 4, 32, 8, 131072
    g = torch.Generator().manual_seed(3)
    k = torch.randn(B, Hkv, N, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(B, Hkv, N, 128, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Hq, 1, 128, generator=g).to(torch.bfloat16)
    c = K.kvc_csm(k.cuda(), v.cuda(), 1, 32, 64, 0.25)
    qd = q.cuda()
    out = K.kvc_decode_attention(qd, c["k_out"], c["v_out"], deg=c["deg_out"])
    assert K.kvc_poll_error() == K.KVC_OK
    o = out.cpu()
    vmax = c["v_out"].float().abs().amax(dim=2).cpu()  # per (b, h, d)
    assert torch.all(torch.isfinite(o))
    assert torch.all(o.abs() <= vmax.repeat_interleave(4, dim=1).unsqueeze(2) + 1e-6)
    kc, vc, dc = c["k_out"].cpu(), c["v_out"].cpu(), c["deg_out"].cpu()
    for b, h in [(0, 0), (1, 5), (2, 3), (3, 7)]:
        check_attention(o[b:b + 1, 4 * h:4 * h + 4].numpy(), q[b:b + 1, 4 * h:4 * h + 4], kc[b:b + 1, h:h + 1],
                        vc[b:b + 1, h:h + 1], dc[b:b + 1, h:h + 1].numpy())


def test_decode_arguments(K):
    q = torch.zeros(1, 18, 1, 128, device="cuda", dtype=torch.bfloat16)
    k = torch.zeros(1, 2, 10, 128, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(K.KvcError):  # 9 query rows per KV head
        K.kvc_decode_attention(q, k, k)
    with pytest.raises(K.KvcError):  # n > capacity
        K.kvc_decode_attention(q[:, :8], k, k, n=11)
    with pytest.raises(K.KvcError):  # a round is never in place
        K.kvc_csm(k, k.clone(), 1, 2, 4, 0.25, out={"k_out": k, "v_out": k.clone(),
                                                  "deg_out": torch.empty(1, 2, 10, dtype=torch.int32, device="cuda"),
                                                  "pos_out": torch.empty(1, 2, 10, dtype=torch.int32, device="cuda")})
    assert K.kvc_poll_error() == K.KVC_OK


def test_append_and_strided_round(K):
    g = torch.Generator().manual_seed(11)
    B, H, cap, n0, t = 2, 3, 700, 500, 37
    k0 = torch.randn(B, H, n0, 128, generator=g).to(torch.bfloat16)
    v0 = torch.randn(B, H, n0, 128, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, H, t, 128, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, H, t, 128, generator=g).to(torch.bfloat16)
    kc = torch.full((B, H, cap, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full((B, H, cap, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    dc = torch.full((B, H, cap), -7, dtype=torch.int32, device="cuda")
    pc = torch.full((B, H, cap), -7, dtype=torch.int32, device="cuda")
    K.kvc_append(kc, vc, 0, k0.cuda(), v0.cuda(), deg_cache=dc, pos_cache=pc, pos0=0)
    K.kvc_append(kc, vc, n0, kn.cuda(), vn.cuda(), deg_cache=dc, pos_cache=pc, pos0=1000)
    n = n0 + t
    assert torch.equal(kc[:, :, :n].cpu(), torch.cat([k0, kn], dim=2))
    assert torch.equal(vc[:, :, :n].cpu(), torch.cat([v0, vn], dim=2))
    assert torch.all(dc[:, :, :n] == 1) and torch.all(dc[:, :, n:] == -7)
    want_pos = torch.cat([torch.arange(n0), torch.arange(1000, 1000 + t)]).int()
    assert torch.equal(pc[:, :, :n].cpu(), want_pos.expand(B, H, n))
    assert torch.isnan(kc[:, :, n:].float()).all()
    # a strided round equals the dense round on the same rows, positions carried through
    dense = K.kvc_csm(kc[:, :, :n].contiguous(), vc[:, :, :n].contiguous(), 2, 9, 16, 0.3,
                      deg=dc[:, :, :n].contiguous())
    m = K.kvc_csm_merges(n, 2, 9, 16, 0.3)
    out = {"k_out": torch.zeros_like(kc), "v_out": torch.zeros_like(vc), "deg_out": torch.zeros_like(dc),
           "pos_out": torch.zeros_like(pc)}
    K.kvc_csm(kc, vc, 2, 9, 16, 0.3, deg=dc, n=n, pos=pc, out=out)
    assert K.kvc_poll_error() == K.KVC_OK
    assert torch.equal(out["k_out"][:, :, :n - m], dense["k_out"])
    assert torch.equal(out["v_out"][:, :, :n - m], dense["v_out"])
    assert torch.equal(out["deg_out"][:, :, :n - m], dense["deg_out"])
    assert torch.equal(out["pos_out"][:, :, :n - m].cpu(), want_pos[dense["pos_out"].long().cpu()])


def test_centroid_cache_decode_loop(K):
    from long_context_kv_kvc_b200.centroid_cache import CentroidCache
    g = torch.Generator().manual_seed(21)
    B, H, Hq, N0, steps = 1, 2, 8, 900, 40
    S, w, chunk, r_init, delta, gap, budget = 2, 16, 16, 0.4, 0.1, 8, 300
    cc = CentroidCache(B, H, 2048, budget=budget, n_sink=S, window=w, chunk=chunk, r_init=r_init, delta=delta, g=gap)
    k0 = torch.randn(B, H, N0, 128, generator=g).to(torch.bfloat16)
    v0 = torch.randn(B, H, N0, 128, generator=g).to(torch.bfloat16)

    def snapshot():
        vw = cc.view()
        return {x: vw[x].cpu().clone() for x in vw}

    def check_round(before, ratio):
        after = snapshot()
        for b in range(B):
            for h in range(H):
                idx = np.searchsorted(before["pos"][b, h].numpy(), after["pos"][b, h].numpy())
                check_row(before["k"][b, h], before["v"][b, h], before["deg"][b, h].numpy(), after["k"][b, h],
                          after["v"][b, h], after["deg"][b, h].numpy(), idx, S, w, chunk, ratio, torch.bfloat16)
        return after

    before = {"k": k0, "v": v0, "deg": torch.ones(B, H, N0, dtype=torch.int32),
              "pos": torch.arange(N0, dtype=torch.int32).expand(B, H, N0)}
    m = cc.prefill(k0.cuda(), v0.cuda())
    r0 = K.kvc_csm_ratio(r_init, delta, 0)  # the fp32 ratio the library merges with
    assert m == O.csm_merges(N0, S, w, chunk, r0) and cc.n == N0 - m and cc.round == 1
    check_round(before, r0)
    rounds = 1
    for s in range(1, steps + 1):
        q = torch.randn(B, Hq, 1, 128, generator=g).to(torch.bfloat16)
        kn = torch.randn(B, H, 1, 128, generator=g).to(torch.bfloat16)
        vn = torch.randn(B, H, 1, 128, generator=g).to(torch.bfloat16)
        pre = snapshot()
        n_before = cc.n
        out = cc.step(q.cuda(), kn.cuda(), vn.cuda())
        # attention over the cache with the new token appended (before any round)
        kk = torch.cat([pre["k"], kn], dim=2)
        vv = torch.cat([pre["v"], vn], dim=2)
        dd = torch.cat([pre["deg"], torch.ones(B, H, 1, dtype=torch.int32)], dim=2)
        check_attention(out.cpu().numpy(), q, kk, vv, dd.numpy())
        if s % gap == 0 and n_before + 1 > budget:
            ratio = K.kvc_csm_ratio(r_init, delta, rounds)
            assert ratio == pytest.approx(O.csm_ratio(r_init, delta, rounds), abs=1e-6)
            rounds += 1
            check_round({"k": kk, "v": vv, "deg": dd,
                         "pos": torch.cat([pre["pos"], torch.full((B, H, 1), N0 + s - 1, dtype=torch.int32)], dim=2)},
                        ratio)
        assert cc.round == rounds
        vw = cc.view()
        assert torch.all(vw["deg"].sum(dim=-1) == N0 + s)  # every token seen is in exactly one centroid
        assert torch.all(vw["pos"][..., 1:] > vw["pos"][..., :-1])
    assert K.kvc_poll_error() == K.KVC_OK
