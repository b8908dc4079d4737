"""The C ABI without a GPU: the library loads, exports every symbol the header declares,
its struct layout matches the C compiler's, and argument validation returns the
documented status codes before anything touches the device."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvc.h")


@pytest.fixture(scope="module")
def K():
    from long_context_kv_kvc_b200 import build
    build.build()
    from long_context_kv_kvc_b200 import kvc
    return kvc


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"KVC_API\s+[\w\s\*]+?\b(kvc_\w+)\s*\(", text)


def test_exports_every_declared_symbol(K):
    names = declared_symbols()
    assert len(names) >= 12
    out = subprocess.check_output(["nm", "-D", "--defined-only", K.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert hasattr(K.lib, n)
    assert set(names) == set(K.EXPORTED)


def test_checks_build_exports_the_same_symbols_and_says_so(K):
    """libkvc_checks.so (KVC_CHECKS=1) is the same ABI; kvc_checks_enabled tells the builds apart."""
    from long_context_kv_kvc_b200 import build
    path = build.build(checks=True)
    out = subprocess.check_output(["nm", "-D", "--defined-only", path], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(declared_symbols()) <= exported
    for lib_path, want in ((path, 1), (build.LIB, 0)):
        L = ctypes.CDLL(lib_path)
        L.kvc_checks_enabled.restype = ctypes.c_int32
        assert L.kvc_checks_enabled() == want
    L = ctypes.CDLL(path)
    L.kvc_status_string.restype = ctypes.c_char_p
    L.kvc_status_string.argtypes = [ctypes.c_int]
    assert b"range check" in L.kvc_status_string(K.KVC_ERR_CHECK)


def test_params_layout_matches_c(K, tmp_path):
    fields = [f[0] for f in K.Params._fields_]
    src = tmp_path / "layout.c"
    body = "".join(f'printf("%zu ", offsetof(kvc_params, {f}));' for f in fields)
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "kvc.h"\n'
                   f'int main(void){{ printf("%zu ", sizeof(kvc_params)); {body} return 0; }}\n')
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    got = list(map(int, subprocess.check_output([str(exe)], text=True).split()))
    want = [ctypes.sizeof(K.Params)] + [getattr(K.Params, f).offset for f in fields]
    assert got == want


def test_header_compiles_as_c_and_cxx(tmp_path):
    for comp, ext in (("gcc", "c"), ("g++", "cpp")):
        src = tmp_path / f"inc.{ext}"
        src.write_text('#include "kvc.h"\nint main(void){ return (int)KVC_OK; }\n')
        subprocess.check_call([comp, "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                               "-o", str(tmp_path / f"inc_{ext}")])


def _p(K, **kw):
    base = dict(B=1, Hq=32, Hkv=8, N=4096, window=32, dtype=K.KVC_BF16, kv_budget=512)
    base.update(kw)
    return K.make_params(**base)


FAKE = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first


def _compress_status(K, p, ws_bytes=1 << 40, **ptrs):
    args = dict(q=FAKE, k=FAKE, v=FAKE, k_out=FAKE, v_out=FAKE, idx=FAKE, hidden=None, hidden_out=None,
                tsp_idx=None, ws=FAKE)
    args.update(ptrs)
    return K.lib.kvc_compress(ctypes.byref(p), args["q"], args["k"], args["v"], args["k_out"],
                              args["v_out"], args["idx"], args["hidden"], args["hidden_out"],
                              args["tsp_idx"], args["ws"], ws_bytes, None)


def test_validation_codes(K):
    assert _compress_status(K, _p(K, D=64)) == K.KVC_ERR_UNSUPPORTED
    assert _compress_status(K, _p(K, dtype=7)) == K.KVC_ERR_UNSUPPORTED
    assert _compress_status(K, _p(K, scope=5)) == K.KVC_ERR_UNSUPPORTED
    assert _compress_status(K, _p(K, window=64, Hq=32, Hkv=4)) == K.KVC_ERR_UNSUPPORTED  # G*w > 256
    assert _compress_status(K, _p(K, Hq=30)) == K.KVC_ERR_ARG  # Hq % Hkv
    assert _compress_status(K, _p(K, B=0)) == K.KVC_ERR_ARG
    assert _compress_status(K, _p(K, pool_kernel=4)) == K.KVC_ERR_ARG
    assert _compress_status(K, _p(K, N=20, window=20, Hq=8, kv_budget=10)) == K.KVC_ERR_ARG  # window >= N
    assert _compress_status(K, _p(K), q=None) == K.KVC_ERR_ARG
    assert _compress_status(K, _p(K, kv_budget=33)) == K.KVC_ERR_BUDGET  # < S + w + 1
    assert _compress_status(K, _p(K, kv_budget=4097)) == K.KVC_ERR_BUDGET  # > N
    assert _compress_status(K, _p(K), k=ctypes.c_void_p((1 << 20) + 8)) == K.KVC_ERR_ALIGN
    assert _compress_status(K, _p(K), ws=ctypes.c_void_p((1 << 20) + 16)) == K.KVC_ERR_ALIGN
    assert _compress_status(K, _p(K), ws_bytes=100) == K.KVC_ERR_WORKSPACE
    # TSP: buffers required when the rate is set, forbidden otherwise
    assert _compress_status(K, _p(K, tsp_rate=0.2, hidden_dim=4096)) == K.KVC_ERR_ARG
    assert _compress_status(K, _p(K), hidden=FAKE) == K.KVC_ERR_ARG
    assert _compress_status(K, _p(K, tsp_rate=1e-5, hidden_dim=4096), hidden=FAKE, hidden_out=FAKE,
                            tsp_idx=FAKE) == K.KVC_ERR_BUDGET  # floor(rate * N) == 0
    assert _compress_status(K, _p(K, tsp_rate=0.2, hidden_dim=4100), hidden=FAKE, hidden_out=FAKE,
                            tsp_idx=FAKE) == K.KVC_ERR_ALIGN  # 8200-byte rows
    p = _p(K)
    p.reserved = 1
    assert _compress_status(K, p) == K.KVC_ERR_ARG


def test_other_entry_points_validate(K):
    L = K.lib
    assert L.kvc_topk(FAKE, 1, 1, 100, 1, 8, 9, FAKE, None, 0, None) == K.KVC_ERR_BUDGET
    assert L.kvc_topk(FAKE, 1, 1, 100, 1, 8, 101, FAKE, None, 0, None) == K.KVC_ERR_BUDGET
    assert L.kvc_topk(None, 1, 1, 100, 1, 8, 20, FAKE, None, 0, None) == K.KVC_ERR_ARG
    assert L.kvc_pool(FAKE, FAKE, 1, 1, 100, 0, 100, 7, None) == K.KVC_ERR_ARG  # in == out
    assert L.kvc_pool(FAKE, ctypes.c_void_p(1 << 21), 1, 1, 100, 0, 100, 6, None) == K.KVC_ERR_ARG
    assert L.kvc_pool(FAKE, ctypes.c_void_p(1 << 21), 1, 1, 100, 50, 40, 7, None) == K.KVC_ERR_ARG
    assert L.kvc_accumulate(FAKE, FAKE, 1, 6, 4, 10, None) == K.KVC_ERR_ARG
    assert L.kvc_gather(FAKE, 1, 8, 100, 24, FAKE, 1, 10, FAKE, None) == K.KVC_ERR_ALIGN
    assert L.kvc_gather(FAKE, 1, 8, 100, 256, FAKE, 3, 10, FAKE, None) == K.KVC_ERR_ARG
    p = _p(K)
    assert L.kvc_score(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, 10, None) == K.KVC_ERR_WORKSPACE
    n = ctypes.c_size_t()
    assert L.kvc_workspace_size(None, ctypes.byref(n)) == K.KVC_ERR_ARG


def test_workspace_size_scales(K):
    small = K.kvc_workspace_size(_p(K))
    big = K.kvc_workspace_size(_p(K, N=131072, B=4, kv_budget=4096))
    assert 0 < small < big
    # compress needs the score rows and their pooled copy at least
    assert big >= 2 * 4 * 8 * 131072 * 4


def test_tsp_count_matches_oracle(K, oracle_lib):
    import numpy as np
    for N, w, S, rate in [(65536, 32, 1, 0.2), (100, 10, 1, 0.0), (100, 10, 1, 0.001), (100, 10, 1, 1.0),
                          (1000, 8, 4, 0.37), (131072, 32, 0, 0.05)]:
        r32 = float(np.float32(rate))
        assert K.kvc_tsp_count(N, w, S, r32) == oracle_lib.tsp_count(N, w, S, r32)


def test_status_strings(K):
    for st in range(0, 9):
        assert len(K.kvc_status_string(st)) >= 2
    assert "unknown" in K.kvc_status_string(99)
    assert K.kvc_version().startswith("kvc ")


def test_next_rows_validate_on_host(K, oracle_lib):
    # every call below fails validation on the host: none reaches a launch with the fake pointers
    L = K.lib
    F2 = ctypes.c_void_p((1 << 20) + 4096)  # a second distinct fake buffer
    sz = ctypes.c_size_t
    # Chunked Soft Matching: merge count, workspace, argument checks
    for args in [(1000, 1, 32, 64, 0.25), (777, 0, 0, 2, 0.5), (515, 1, 3, 6, 0.45), (40, 5, 35, 16, 0.5),
                 (130, 1, 1, 2, 0.5), (9, 0, 0, 4, 0.5)]:
        assert K.kvc_csm_merges(*args) == oracle_lib.csm_merges(*args)
    assert L.kvc_csm_merges(100, 1, 8, 3, 0.25) == -1      # odd chunk
    assert L.kvc_csm_merges(100, 1, 8, 130, 0.25) == -1    # chunk > 128
    assert L.kvc_csm_merges(100, 1, 8, 16, 0.6) == -1      # ratio > 0.5
    n = sz()
    assert L.kvc_csm_workspace_size(1, 2, 1000, 1, 32, 64, ctypes.c_float(0.25), ctypes.byref(n)) == K.KVC_OK
    assert n.value > 0
    def csm(k=FAKE, v=F2, ko=ctypes.c_void_p(1 << 22), vo=ctypes.c_void_p(1 << 23), N=1000, ld_in=0, ld_out=0,
            D=128, dtype=K.KVC_BF16, chunk=64, ratio=0.25, ws_bytes=1 << 40):
        return L.kvc_csm(k, v, None, None, 1, 2, N, ld_in, D, dtype, 1, 32, chunk, ctypes.c_float(ratio), ko, vo,
                         FAKE, FAKE, ld_out, FAKE, ws_bytes, None)
    assert csm(k=None) == K.KVC_ERR_ARG
    assert csm(ko=FAKE) == K.KVC_ERR_ARG                   # in place
    assert csm(chunk=7) == K.KVC_ERR_ARG
    assert csm(ld_in=999) == K.KVC_ERR_ARG                 # capacity below N
    assert csm(D=64) == K.KVC_ERR_UNSUPPORTED
    assert csm(dtype=9) == K.KVC_ERR_UNSUPPORTED
    assert csm(k=ctypes.c_void_p((1 << 20) + 8)) == K.KVC_ERR_ALIGN
    assert csm(ws_bytes=10) == K.KVC_ERR_WORKSPACE
    # append
    assert L.kvc_append(FAKE, F2, None, None, 1, 2, 100, 90, FAKE, F2, 11, 0, 128, K.KVC_BF16, None) == K.KVC_ERR_ARG
    assert L.kvc_append(FAKE, F2, None, None, 1, 2, 100, 90, FAKE, F2, 5, 0, 64, K.KVC_BF16, None) == \
        K.KVC_ERR_UNSUPPORTED
    # decode attention
    def dec(q=FAKE, Hq=32, Hkv=8, nq=1, n=1000, ld=0, D=128, dtype=K.KVC_BF16, ws_bytes=1 << 40):
        return L.kvc_decode_attention(q, FAKE, F2, None, 1, Hq, Hkv, nq, n, ld, D, dtype, FAKE, FAKE, ws_bytes, None)
    assert dec(q=None) == K.KVC_ERR_ARG
    assert dec(Hq=30) == K.KVC_ERR_ARG                     # Hq % Hkv
    assert dec(nq=3) == K.KVC_ERR_UNSUPPORTED              # 12 query rows per KV head
    assert dec(ld=999) == K.KVC_ERR_ARG                    # capacity below n
    assert dec(D=64) == K.KVC_ERR_UNSUPPORTED
    assert dec(q=ctypes.c_void_p((1 << 20) + 8)) == K.KVC_ERR_ALIGN
    assert dec(ws_bytes=10) == K.KVC_ERR_WORKSPACE
    small, big = K.kvc_decode_attention_workspace_size(1, 32, 8, 1, 1000), \
        K.kvc_decode_attention_workspace_size(4, 32, 8, 1, 98313)
    assert 0 < small <= big
    # sequence sharding and the distributed select
    p = _p(K)
    assert L.kvc_shard_workspace_size(ctypes.byref(_p(K, scope=K.KVC_SCOPE_ALL_HEADS)), 100, ctypes.byref(n)) == \
        K.KVC_ERR_UNSUPPORTED
    assert L.kvc_shard_workspace_size(ctypes.byref(p), 100, ctypes.byref(n)) == K.KVC_OK and n.value > 0
    assert L.kvc_shard_stats(ctypes.byref(p), FAKE, FAKE, 100, 4000, FAKE, FAKE, 1 << 40, None) == K.KVC_ERR_ARG
    assert L.kvc_shard_stats(ctypes.byref(p), FAKE, FAKE, 100, 0, FAKE, FAKE, 10, None) == K.KVC_ERR_WORKSPACE
    assert L.kvc_shard_scores(ctypes.byref(p), FAKE, FAKE, 100, 0, FAKE, 0, FAKE, FAKE, 1 << 40, None) == \
        K.KVC_ERR_ARG                                      # no shards
    assert L.kvc_select_hist(FAKE, 2, 100, 0, 100, FAKE, 0, 13, FAKE, None) == K.KVC_ERR_ARG  # 13-bit digit
    assert L.kvc_select_hist(FAKE, 2, 100, 0, 100, FAKE, 22, 11, FAKE, None) == K.KVC_ERR_ARG  # 33 bits
    assert L.kvc_select_hist(FAKE, 2, 100, 50, 40, FAKE, 0, 11, FAKE, None) == K.KVC_ERR_ARG   # lo > hi
    assert L.kvc_select_emit(FAKE, 2, 100, 0, 100, FAKE, FAKE, -1, FAKE, 100, FAKE, None) == K.KVC_ERR_ARG


def test_binding_rejects_mixed_dtypes(K):
    import torch
    q = torch.zeros(1, 4, 1, 128, dtype=torch.float32)
    k = torch.zeros(1, 1, 10, 128, dtype=torch.bfloat16)
    with pytest.raises(K.KvcError):
        K.kvc_decode_attention(q, k, k)
    with pytest.raises(K.KvcError):
        K.kvc_csm(k, k.float(), 1, 2, 4, 0.25)
    with pytest.raises(K.KvcError):
        K.kvc_append(k, k, 0, k.float(), k.float())
