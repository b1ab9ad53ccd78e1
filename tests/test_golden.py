"""The oracle against its frozen regression record (CPU only).

``tests/golden/oracle_regression.json`` holds the oracle's results on small seeded cases,
written by ``tests/golden/make_oracle_regression.py`` from ``oracle/`` alone.  The pages print
no worked numerical example, so the record is not a page value: it pins the oracle to its own
earlier, pinned state, so that any change to its arithmetic is a visible diff.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "golden"))

import make_oracle_regression as mor  # noqa: E402


def test_oracle_matches_regression_record():
    with open(mor.OUT) as fh:
        rec = json.load(fh)
    assert rec["shapes"]["seed"] == mor.SEED
    got = mor.results()
    assert set(got) == set(rec["arrays"])
    for name, a in got.items():
        entry = rec["arrays"][name]
        assert list(a.shape) == entry["shape"], name
        if "hex" in entry:
            # outputs pass through exp(): compare to 1e-14 of the largest magnitude, so that
            # a libm whose exp differs in the last place still agrees
            want = np.array([float.fromhex(h) for h in entry["hex"]]).reshape(a.shape)
            scale = max(float(np.max(np.abs(want))), 1e-300)
            assert float(np.max(np.abs(a - want))) <= 1e-14 * scale, name
        else:
            # caches, lengths and counts involve no transcendental: bit-exact
            assert mor.sha(a) == entry["sha256"], name
