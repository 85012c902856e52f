"""The oracle still reproduces its stored fixture (tests/golden/make_golden.py)."""
import os

import numpy as np

from tests.golden.make_golden import compute

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    res = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, *vals = line.split()
            res[key] = np.array([float(x) for x in vals])
    return res


def test_tiny_tree8_d32_fixture():
    want = _load("tiny_tree8_d32.txt")
    got = compute()
    assert set(want) == set(got)
    for key in want:
        np.testing.assert_allclose(got[key], want[key], rtol=1e-13, atol=1e-15, err_msg=key)
