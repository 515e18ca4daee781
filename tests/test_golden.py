"""The oracle reproduces the fixtures under tests/golden/ (a regression guard against unintended
change of the oracle, written by make_golden.py from the oracle and the seeded generator only --
these are not pins, the pins are the test_oracle_* tests).  Codes, scales and the
per-tensor scales must match exactly; float64 outputs to 1e-12 relative (a matmul's last
bits depend on the BLAS build)."""

import json
import os
import sys

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_golden  # noqa: E402


@pytest.mark.parametrize("name", sorted(make_golden.FIXTURES))
def test_oracle_reproduces_the_fixture(name):
    with open(os.path.join(HERE, "golden", name)) as f:
        stored = json.load(f)
    now = make_golden.FIXTURES[name]()
    assert now.keys() == stored.keys()
    for key in now:
        if key == "y_hex":
            a = np.array([float.fromhex(v) for v in now[key]])
            b = np.array([float.fromhex(v) for v in stored[key]])
            assert np.allclose(a, b, rtol=1e-12, atol=1e-300)
        else:
            assert now[key] == stored[key], key
