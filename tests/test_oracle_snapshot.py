"""The fp64 oracle against its stored regression snapshot (tests/golden/): kept
sets and candidate counts bit-exact, outputs to 1e-12 relative. The snapshot was
written by tests/golden/make_oracle_snapshot.py from oracle/ alone; the oracle's
correctness itself is pinned in test_oracle_pins.py."""
import json
import os

import numpy as np

from tests.golden import make_oracle_snapshot as M

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_tiny_snapshot.json")


def test_oracle_matches_snapshot():
    want = json.load(open(GOLD))
    got = M.compute()
    assert got["intervals"] == want["intervals"]
    assert got["nq"] == want["nq"]
    assert got["nkept"] == want["nkept"]
    assert got["kept"] == want["kept"]
    for (ix, v), (ix2, v2) in zip(got["out_samples"], want["out_samples"]):
        assert ix == ix2
        assert abs(v - v2) <= 1e-12 * max(1.0, abs(v2))
    assert np.isclose(got["out_abs_sum"], want["out_abs_sum"], rtol=1e-12, atol=0)
