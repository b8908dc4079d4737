"""kvc_score_noalloc: scoring without a caller workspace.

Some callers cannot allocate device memory where compaction runs (an engine that has
already handed all of device memory to its own pool, or a plugin interface that forbids
cudaMalloc/cudaFree during a step).  This entry point keeps its scratch in a fixed array
inside the library instead.  The test calls it through the C ABI twice in a row, on
different inputs, and checks each result against kvc_score (which uses a caller
workspace) within the score tolerance of the other parity tests, and against the fp64
oracle.  It lives in its own file, named so that pytest collects it last.
"""
import pytest
import torch

from long_context_kv_kvc_b200 import synth
from oracle import oracle as O
from parity_util import SCORE_RTOL, check_scores

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


def _scores_both_ways(K, wl):
    inp = synth.make_inputs(wl, with_v=False)
    q, k = inp["q"].cuda(), inp["k"].cuda()
    p = K.params_for(wl)
    Hs = wl.Hkv if wl.scope == K.KVC_SCOPE_PER_KV_HEAD else 1
    ws = torch.empty(K.kvc_workspace_size(p), dtype=torch.uint8, device="cuda")
    with_ws = torch.empty((wl.B, Hs, wl.N), dtype=torch.float32, device="cuda")
    K.kvc_score(p, q, k, with_ws, ws)
    no_ws = torch.full((wl.B, Hs, wl.N), float("nan"), dtype=torch.float32, device="cuda")
    K.kvc_score_noalloc(p, q, k, no_ws)
    assert K.kvc_poll_error() == K.KVC_OK
    ref = O.score(inp["q"], inp["k"], window=wl.window, scope=wl.scope)
    return no_ws.double().cpu().numpy(), with_ws.double().cpu().numpy(), ref


def test_noalloc_matches_workspace_entry_point_twice(K):
    first = synth.scaled(synth.LLAMA8B_32K, B=2, N=5003, n_hubs=32)
    second = synth.scaled(synth.STRUCTKV_8L_32K, N=3001, n_layers=2, kv_budget=300, n_hubs=16,
                          seeds=(7,))
    for wl in (first, second):
        got, want, ref = _scores_both_ways(K, wl)
        check_scores(got, want, rtol=SCORE_RTOL)
        check_scores(got, ref, rtol=SCORE_RTOL)


def test_noalloc_rejects_what_does_not_fit(K):
    # no buffers at all: the size check must reject the call before anything is touched
    wl = synth.LLAMA8B_128K_B4.replace(n_layers=2)
    p = K.params_for(wl)
    with pytest.raises(K.KvcError) as e:
        K.kvc_score_noalloc(p, None, None, None)
    assert e.value.status == K.KVC_ERR_WORKSPACE
