"""Regression snapshot of the oracle (tests/golden/tiny_regression.json)."""
import json
import os

import numpy as np

from tests.golden.make_golden import compute

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_matches_its_committed_snapshot():
    with open(os.path.join(HERE, "golden", "tiny_regression.json")) as f:
        want = json.load(f)
    got = compute()
    assert got["idx"] == want["idx"]
    for key in ("scores_row39", "out_row39_head0_first8", "lse_row39"):
        np.testing.assert_allclose(got[key], want[key], rtol=1e-12, atol=1e-12)
