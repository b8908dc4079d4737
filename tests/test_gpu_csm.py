"""Parity of Chunked Soft Matching (kvc_csm) through the C ABI with the fp64 oracle.

Cosine similarities are fp32 on the GPU and fp64 in the oracle, so the decisions they take
follow the band rule used for the top-k: a match whose oracle similarity is clearly above
(below) the m-th best must (must not) merge; only matches within 1e-5 of it may differ.
Given the GPU's merge set, every kept row must equal the exact degree-weighted mean of the
same tokens up to fp32 summation error (2e-6 of the summands' magnitude) plus, for bf16
outputs, half a unit in the last place; every unmerged row must be a bit-exact copy, and
degrees and positions must be exact.  When the GPU's merge set is the oracle's (the common
case), the kept rows are also compared with the oracle's own rounded outputs (one unit in
the last place for bf16) and the bit-identical fraction is reported.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from parity_util import check_csm_row as check_row

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


def make_kv(B, H, N, dtype, seed, dup=0, zero=0):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, H, N, 128, generator=g)
    v = torch.randn(B, H, N, 128, generator=g)
    if dup:
        # planted near-duplicates: some tokens repeat their left neighbour's key direction
        idx = torch.randint(1, N - 1, (dup,), generator=g)
        k[:, :, idx] = 1.5 * k[:, :, idx - 1]
    if zero:
        # zero keys: similarity 0 with every token
        k[:, :, torch.randint(0, N, (zero,), generator=g)] = 0.0
    return k.to(dtype), v.to(dtype)


# bf16 keys take the tensor-core match (128-token tiles holding whole chunks: 128 for chunk
# 2, 64 and 128, 126 for chunk 6, 96 for chunk 48), fp32 keys the CUDA-core one
CASES = [
    dict(B=1, H=2, N=1000, S=1, w=32, chunk=64, ratio=0.25, dtype=torch.bfloat16, deg=False, dup=40, zero=0),
    dict(B=2, H=1, N=777, S=0, w=0, chunk=2, ratio=0.5, dtype=torch.float32, deg=True, dup=0, zero=0),
    dict(B=1, H=3, N=2053, S=4, w=16, chunk=128, ratio=0.1, dtype=torch.bfloat16, deg=True, dup=100, zero=0),
    dict(B=1, H=1, N=515, S=1, w=3, chunk=6, ratio=0.45, dtype=torch.float32, deg=False, dup=20, zero=6),
    dict(B=1, H=2, N=700, S=3, w=5, chunk=6, ratio=0.3, dtype=torch.bfloat16, deg=True, dup=30, zero=8),
    dict(B=2, H=1, N=1500, S=0, w=0, chunk=48, ratio=0.2, dtype=torch.bfloat16, deg=False, dup=50, zero=0),
    dict(B=1, H=1, N=401, S=2, w=7, chunk=2, ratio=0.5, dtype=torch.bfloat16, deg=True, dup=0, zero=0),
    dict(B=1, H=1, N=300, S=130, w=140, chunk=16, ratio=0.5, dtype=torch.bfloat16, deg=False, dup=5, zero=0),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_csm_matches_oracle(K, case):
    c = CASES[case]
    B, H, N = c["B"], c["H"], c["N"]
    k, v = make_kv(B, H, N, c["dtype"], 30 + case, dup=c["dup"], zero=c["zero"])
    deg = (torch.randint(1, 6, (B, H, N), generator=torch.Generator().manual_seed(case), dtype=torch.int32)
           if c["deg"] else torch.ones((B, H, N), dtype=torch.int32))
    out = K.kvc_csm(k.cuda(), v.cuda(), c["S"], c["w"], c["chunk"], c["ratio"],
                    deg=deg.cuda() if c["deg"] else None)
    assert K.kvc_poll_error() == K.KVC_OK
    same = []
    for b in range(B):
        for h in range(H):
            same.append(check_row(k[b, h], v[b, h], deg[b, h].numpy(), out["k_out"][b, h].cpu(),
                                  out["v_out"][b, h].cpu(), out["deg_out"][b, h].cpu().numpy(),
                                  out["pos_out"][b, h].cpu().numpy(), c["S"], c["w"], c["chunk"], c["ratio"],
                                  c["dtype"]))
    compared = [f for f in same if f is not None]
    print(f"case {case}: {len(compared)}/{len(same)} rows with the oracle's merge set, bit-identical elements "
          f"{(sum(compared) / len(compared)) if compared else float('nan'):.4f}")
    if not c["zero"]:
        # (zero keys tie at cosine 0 with every token, which leaves their rows ambiguous)
        assert compared, "no row merged exactly the oracle's tokens"


EDGE_CASES = [
    # sinks and window cover the row: no candidate, the round is the identity
    dict(N=40, S=5, w=35, chunk=16, ratio=0.5),
    # one chunk shorter than the chunk size, odd length
    dict(N=50, S=2, w=9, chunk=64, ratio=0.3),
    # every matchable A token merges (m = n_A: even |C|, chunks of 2, r = 0.5)
    dict(N=130, S=1, w=1, chunk=2, ratio=0.5),
    # every A merges with chunks of 128 (one ragged last chunk)
    dict(N=400, S=0, w=3, chunk=128, ratio=0.5),
]


@pytest.mark.parametrize("case", range(len(EDGE_CASES)))
def test_csm_edge_cases(K, case):
    c = EDGE_CASES[case]
    N, S, w, chunk, ratio = c["N"], c["S"], c["w"], c["chunk"], c["ratio"]
    for dtype in (torch.bfloat16, torch.float32):
        k, v = make_kv(1, 2, N, dtype, 50 + case, dup=5)
        deg = torch.randint(1, 4, (1, 2, N), generator=torch.Generator().manual_seed(case), dtype=torch.int32)
        out = K.kvc_csm(k.cuda(), v.cuda(), S, w, chunk, ratio, deg=deg.cuda())
        assert K.kvc_poll_error() == K.KVC_OK
        m = O.csm_merges(N, S, w, chunk, K.kvc_csm_ratio(ratio, 0.0, 0))
        assert out["pos_out"].shape[-1] == N - m
        for h in range(2):
            check_row(k[0, h], v[0, h], deg[0, h].numpy(), out["k_out"][0, h].cpu(), out["v_out"][0, h].cpu(),
                      out["deg_out"][0, h].cpu().numpy(), out["pos_out"][0, h].cpu().numpy(), S, w, chunk, ratio,
                      dtype)


def test_csm_identity_and_arguments(K):
    k, v = make_kv(1, 2, 300, torch.bfloat16, 7)
    out = K.kvc_csm(k.cuda(), v.cuda(), 1, 8, 16, 0.0)
    assert torch.equal(out["k_out"].cpu(), k) and torch.equal(out["v_out"].cpu(), v)
    assert torch.equal(out["pos_out"].cpu(), torch.arange(300, dtype=torch.int32).expand(1, 2, 300))
    assert torch.all(out["deg_out"] == 1)
    assert K.kvc_csm_merges(10, 1, 2, 4, 0.5) == O.csm_merges(10, 1, 2, 4, 0.5) == 3
    assert K.kvc_csm_merges(9, 0, 0, 4, 0.5) == O.csm_merges(9, 0, 0, 4, 0.5) == 4
    assert K.kvc_csm_ratio(0.5, 0.1, 2) == pytest.approx(O.csm_ratio(0.5, 0.1, 2))
    for bad in [dict(chunk=3), dict(chunk=130), dict(ratio=0.6)]:
        a = dict(chunk=16, ratio=0.25)
        a.update(bad)
        with pytest.raises(K.KvcError):
            K.kvc_csm(k.cuda(), v.cuda(), 1, 8, a["chunk"], a["ratio"])
    assert K.kvc_poll_error() == K.KVC_OK


def test_csm_full_size_128k_batch4(K):
    """The 8B shape at 128K x 4 (bf16 K and V, 32 rows): invariants on every row, the band
    rule and the kept rows against the oracle on two sampled rows."""
    B, H, N, S, w, chunk, ratio = 4, 8, 131072, 1, 32, 64, 0.25
    k, v = make_kv(B, H, N, torch.bfloat16, 99, dup=2000)
    kd, vd = k.cuda(), v.cuda()
    out = K.kvc_csm(kd, vd, S, w, chunk, ratio)
    assert K.kvc_poll_error() == K.KVC_OK
    m = O.csm_merges(N, S, w, chunk, ratio)
    n_out = N - m
    pos = out["pos_out"]
    assert pos.shape == (B, H, n_out)
    assert torch.all(pos[..., 1:] > pos[..., :-1])
    assert torch.all(out["deg_out"].sum(dim=-1) == N)
    assert torch.all(pos[..., :S] == torch.arange(S, device="cuda"))
    assert torch.all(pos[..., -w:] == torch.arange(N - w, N, device="cuda", dtype=torch.int32))
    # rows of degree 1 are exact copies of their source rows
    single = out["deg_out"] == 1
    src = torch.gather(kd, 2, pos.long().unsqueeze(-1).expand(-1, -1, -1, 128))
    assert torch.equal(out["k_out"][single], src[single])
    for b, h in [(0, 0), (3, 7)]:
        check_row(k[b, h], v[b, h], np.ones(N, np.int32), out["k_out"][b, h].cpu(), out["v_out"][b, h].cpu(),
                  out["deg_out"][b, h].cpu().numpy(), out["pos_out"][b, h].cpu().numpy(), S, w, chunk, ratio,
                  torch.bfloat16)
