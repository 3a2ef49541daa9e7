"""The oracle still reproduces its stored fixtures (regression pin against drift)."""
import json
import os

import numpy as np
import pytest

from tests.golden.make_golden import NAMES, expected_actions

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


@pytest.mark.parametrize("name", NAMES)
def test_oracle_matches_fixture(name):
    with open(os.path.join(HERE, f"{name}_actions.json")) as f:
        d = json.load(f)
    ref = np.array(d["actions"]).reshape(d["shape"])
    got = expected_actions(name)
    assert got.shape == ref.shape
    assert np.allclose(got, ref, rtol=0, atol=1e-12)
