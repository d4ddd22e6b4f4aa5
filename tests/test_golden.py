"""The oracle still reproduces its stored tiny-layer values (tests/golden)."""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_tiny  # noqa: E402


def test_oracle_reproduces_tiny_golden():
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        want = json.load(f)
    got = make_tiny.compute()
    assert got["rows"] == want["rows"]
    np.testing.assert_array_equal(np.array(got["idx"]), np.array(want["idx"]))
    np.testing.assert_allclose(got["score_sums"], want["score_sums"], rtol=1e-12)
    np.testing.assert_allclose(np.array(got["O"]), np.array(want["O"]), rtol=0, atol=1e-11)
    np.testing.assert_allclose(np.array(got["lse"]), np.array(want["lse"]), rtol=0, atol=1e-11)
