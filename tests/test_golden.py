"""The oracle still reproduces its frozen CG table (tests/golden/)."""
import os

import numpy as np

from oracle.cg import real_cg

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "real_cg_natural_l3.txt")


def test_real_cg_matches_frozen_table():
    seen = {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("#"):
                continue
            l1, l2, l3, m1, m2, m3, v = line.split()
            l1, l2, l3, m1, m2, m3 = map(int, (l1, l2, l3, m1, m2, m3))
            seen.setdefault((l1, l2, l3), np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1)))[
                m1 + l1, m2 + l2, m3 + l3] = float(v)
    assert len(seen) == 23
    for (l1, l2, l3), C in seen.items():
        assert np.max(np.abs(real_cg(l1, l2, l3) - C)) < 1e-15
