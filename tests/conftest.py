import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_lib():
    from oracle import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _checks_build_error_word(request):
    """Under KVC_CHECKS=1 (the range-checking library), every GPU test must end with the device
    error word clear: a failed range check anywhere in it surfaces as KVC_ERR_CHECK here.
    Tests that provoke a timeout or a bad index poll (and clear) the word themselves."""
    yield
    if os.environ.get("KVC_CHECKS") != "1" or request.node.get_closest_marker("gpu") is None:
        return
    K = sys.modules.get("long_context_kv_kvc_b200.kvc")
    if K is None:
        return
    assert K.kvc_checks_enabled(), "KVC_CHECKS=1 but the regular library is loaded"
    st = K.kvc_poll_error()
    assert st == K.KVC_OK, f"device error word after the test: {K.kvc_status_string(st)}"
