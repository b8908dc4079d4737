"""CentroidCache's host logic on CPU: when rounds run and with which ratio, how positions
and degrees carry through rounds, capacity and argument errors.  The library calls are
replaced by oracle-backed stand-ins with the same contracts (the GPU test runs the real
kernels)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O


class FakeKvc:
    """kvc_append / kvc_csm / kvc_decode_attention / schedule helpers on CPU tensors."""

    def __init__(self):
        self.rounds = []  # (n before, ratio, merges)

    def kvc_csm_ratio(self, r_init, delta, round_):
        return float(np.float32(O.csm_ratio(r_init, delta, round_)))

    def kvc_csm_merges(self, N, S, w, chunk, ratio):
        return O.csm_merges(N, S, w, chunk, ratio)

    def kvc_csm_workspace_size(self, *args):
        return 0

    def kvc_append(self, k_cache, v_cache, n, k_new, v_new, deg_cache=None, pos_cache=None, pos0=0):
        t = k_new.shape[2]
        k_cache[:, :, n:n + t] = k_new
        v_cache[:, :, n:n + t] = v_new
        deg_cache[:, :, n:n + t] = 1
        pos_cache[:, :, n:n + t] = torch.arange(pos0, pos0 + t, dtype=torch.int32)

    def kvc_csm(self, k, v, S, w, chunk, r, deg=None, n=None, pos=None, out=None, ws=None):
        res = O.csm(k[:, :, :n], v[:, :, :n], deg[:, :, :n].numpy(), n_sink=S, window=w, chunk=chunk, ratio=r)
        keep = n - res["m"]
        out["k_out"][:, :, :keep] = res["k_out"]
        out["v_out"][:, :, :keep] = res["v_out"]
        out["deg_out"][:, :, :keep] = torch.from_numpy(res["deg_out"])
        idx = torch.from_numpy(res["pos_out"]).long()
        out["pos_out"][:, :, :keep] = torch.gather(pos[:, :, :n], 2, idx)
        self.rounds.append((n, r, res["m"]))

    def kvc_decode_attention(self, q, k, v, deg=None, n=None):
        return torch.from_numpy(O.centroid_attention(q, k[:, :, :n], v[:, :, :n], deg[:, :, :n].numpy())).float()


@pytest.fixture
def cache_mod(monkeypatch):
    from long_context_kv_kvc_b200 import centroid_cache
    fake = FakeKvc()
    monkeypatch.setattr(centroid_cache, "kvc", fake)
    return centroid_cache, fake


def test_schedule_rounds_and_ratios(cache_mod):
    cc_mod, fake = cache_mod
    g = torch.Generator().manual_seed(1)
    B, H, Hq, N0, S, w, chunk, gap, budget = 1, 2, 4, 300, 2, 8, 8, 5, 120
    r_init, delta = 0.4, 0.1
    cc = cc_mod.CentroidCache(B, H, 1024, budget=budget, n_sink=S, window=w, chunk=chunk, r_init=r_init,
                              delta=delta, g=gap, dtype=torch.float32, device="cpu")
    k0, v0 = torch.randn(B, H, N0, 128, generator=g), torch.randn(B, H, N0, 128, generator=g)
    m0 = cc.prefill(k0, v0)
    assert fake.rounds[0][:2] == (N0, pytest.approx(r_init)) and m0 == fake.rounds[0][2] and cc.n == N0 - m0
    n, rounds = cc.n, 1
    for s in range(1, 31):
        q = torch.randn(B, Hq, 1, 128, generator=g)
        kn, vn = torch.randn(B, H, 1, 128, generator=g), torch.randn(B, H, 1, 128, generator=g)
        out = cc.step(q, kn, vn)
        assert out.shape == (B, Hq, 1, 128)
        n += 1
        if s % gap == 0 and n > budget:
            r = float(np.float32(O.csm_ratio(r_init, delta, rounds)))
            m = O.csm_merges(n, S, w, chunk, r)
            rounds += 1
            if m > 0:
                assert fake.rounds[-1] == (n, pytest.approx(r), m)
            n -= m
        assert cc.n == n and cc.round == rounds
        vw = cc.view()
        assert torch.all(vw["deg"].sum(-1) == N0 + s)            # every token in one centroid
        assert torch.all(vw["pos"][..., 1:] > vw["pos"][..., :-1])  # positions ascending
        assert torch.equal(vw["pos"][..., :S], torch.arange(S, dtype=torch.int32).expand(B, H, S))
        assert torch.all(vw["pos"][..., -1] == N0 + s - 1)        # the newest token is kept
    assert rounds >= 3  # rounds at steps 5, 10, ... while over budget, until the ratio reaches 0


def test_no_round_under_budget_and_errors(cache_mod):
    cc_mod, fake = cache_mod
    cc = cc_mod.CentroidCache(1, 1, 64, budget=100, n_sink=1, window=4, chunk=4, r_init=0.5, delta=0.1, g=2,
                              dtype=torch.float32, device="cpu")
    k = torch.randn(1, 1, 60, 128)
    assert cc.prefill(k, k.clone()) == 0 and cc.round == 0 and not fake.rounds  # under budget: no round
    with pytest.raises(RuntimeError):
        cc.step(torch.randn(1, 1, 1, 128), torch.randn(1, 1, 5, 128), torch.randn(1, 1, 5, 128))  # 60 + 5 > 64
    with pytest.raises(ValueError):
        cc_mod.CentroidCache(1, 1, 64, budget=10, n_sink=1, window=4, chunk=4, r_init=0.7, delta=0.1, g=2,
                             device="cpu")
