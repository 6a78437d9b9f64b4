"""The oracle reproduces its stored regression fixtures (tests/golden/)."""

import os

import numpy as np
import pytest

from tests.golden import make_golden

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    rows, vals = [], []
    with open(os.path.join(HERE, f"{name}.txt")) as f:
        for line in f:
            if line.startswith("#"):
                continue
            parts = line.split()
            rows.append(int(parts[0]))
            vals.append([float(t) for t in parts[1:]])
    return rows, np.array(vals)


@pytest.mark.parametrize("name", sorted(make_golden.CASES))
def test_oracle_matches_stored_fixture(name):
    rows, stored = load(name)
    _, rows_now, vals = make_golden.compute(name)
    assert rows == list(rows_now)
    np.testing.assert_allclose(vals, stored, rtol=0, atol=1e-12)
