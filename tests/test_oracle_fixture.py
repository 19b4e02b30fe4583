"""The oracle against its own stored results on a tiny seeded case (tests/golden/oracle_toy.json,
written by tests/golden/make_oracle_fixture.py from the oracle alone).

This is a regression pin, not a pin to the pages (they print no worked example): kept sets and
counts must match exactly, floating results to 1e-12.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))


def test_oracle_matches_its_stored_results(oracle_mod):
    import make_oracle_fixture as fx
    with open(os.path.join(HERE, "golden", "oracle_toy.json")) as f:
        want = json.load(f)
    got = fx.compute()
    assert got["case"] == want["case"]
    assert got["kept"] == want["kept"]
    assert got["count"] == want["count"]
    for key in ("mass", "kept_mass", "O_rows"):
        np.testing.assert_allclose(np.array(got[key]), np.array(want[key]), rtol=0, atol=1e-12, err_msg=key)
    lg, lw = np.array(got["lse"]), np.array(want["lse"])
    assert np.array_equal(np.isinf(lg), np.isinf(lw))
    np.testing.assert_allclose(lg[np.isfinite(lg)], lw[np.isfinite(lw)], rtol=0, atol=1e-12)
