"""Fixtures printed by the pages (tests/golden/), each with its citation in the file.

The only worked example with printed numbers (the scrapbox "KV Cache" section)
prints no inputs, so it cannot pin the oracle's values; it records the
last-row invariant, which the oracle pin ``pin_decode_is_last_row`` checks on
the oracle itself.  Here: the page's two printed results agree to the printed
precision."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [np.array([float(x) for x in line.split()]) for line in f
                if line.strip() and not line.startswith("#")]


def test_kv_cache_last_row_fixture():
    full_last, single = _rows("kv_cache_last_row.txt")
    assert full_last.shape == single.shape == (8,)
    np.testing.assert_allclose(single, full_last, rtol=1e-8, atol=1e-8)
