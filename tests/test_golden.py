"""The oracle reproduces its stored regression values (tests/golden/oracle_regression.json).

The pages print no worked example, so these values pin nothing about correctness (the pins
are in test_oracle_pins.py); they make any change to the oracle's arithmetic visible.  A
deliberate change regenerates the file with tests/golden/make_golden.py and names the
passage that justifies it in the commit message."""
import importlib.util
import json
import os

import numpy as np

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load_generator():
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(HERE, "make_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _compare(got, want, path=""):
    if isinstance(want, dict):
        assert set(got) == set(want), path
        for k in want:
            _compare(got[k], want[k], f"{path}.{k}")
    elif isinstance(want, (list, tuple)):
        g, w = np.asarray(got), np.asarray(want)
        assert g.shape == w.shape, path
        if np.issubdtype(w.dtype, np.integer):
            assert np.array_equal(g, w), path
        else:
            np.testing.assert_allclose(g, w, rtol=1e-12, atol=1e-300, err_msg=path)
    elif isinstance(want, float):
        assert abs(got - want) <= 1e-12 * abs(want) + 1e-300, path
    else:
        assert got == want, path


def test_oracle_matches_stored_regression_values():
    with open(os.path.join(HERE, "oracle_regression.json")) as f:
        stored = json.load(f)
    _compare(_load_generator().cases(), stored)
