"""The workloads of the configurations other than the benchmarked one, at their full sizes,
through the C ABI in the launch configuration the benchmark times, against the fp64 oracle
on every score row:

* Llama-3.1-8B head layout at 32K context (32/8 heads, budget 2048 per KV head);
* StructKV cumulative centrality: 8 layers at 32K, scores summed over all layers and heads,
  one global set of 2048 (StructKV page, sec. 1 "Global In-Degree Centrality");
* FastKV: token-selective propagation of the top 20 % by head-summed saliency at 64K with
  4096-wide hidden rows, and separately a KV budget of 1024 per KV head (FastKV page,
  sec. 2A "Token-Selective Propagation" and 2B "Entkoppelte KV-Cache-Reduktion").

Scores within 1e-3 relative at every position, index sets under the band rule, every
gathered K/V and hidden row bit-exact (parity_util.run_case).
"""
import pytest
import torch

from long_context_kv_kvc_b200 import synth
from parity_util import run_case

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


@pytest.mark.parametrize("name", ["llama8b-32k", "structkv-8layer-32k", "fastkv-tsp20-64k"])
def test_full_size_config(K, name):
    wl = synth.WORKLOADS[name]
    out, ref, scores = run_case(K, wl)
    if wl.tsp_rate > 0:
        assert out["hidden_out"].shape == (wl.B, K.kvc_tsp_count(wl.N, wl.window, wl.n_sink, wl.tsp_rate),
                                           wl.hidden_dim)
    torch.cuda.synchronize()
    assert K.kvc_poll_error() == K.KVC_OK
