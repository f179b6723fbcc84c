"""The code-comparison rule every parity claim rests on, pinned on hand-made
cases (host only): a GPU code may differ from the oracle's only by one, and
only where the oracle's v/s lies within 1e-6 relative of the midpoint
between the two codes (round to nearest, CoQuant Eq. (1); the allowance
covers the fp32 summation order of the rotation).  Both the tests' checker
and the benchmark's flip counter follow it; a checker that measured the
distance absolutely, to the wrong midpoint, or let differences of two
through would fail here."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from tests.parity_util import MIDPOINT_REL, check_codes  # noqa: E402


def _case():
    # oracle codes and the values v/s they were rounded from (one token row
    # of 32 codes: the packed layout's group size)
    q = np.array([[0, 2, -3, 7, -7, 1, 0, -1] * 4], dtype=np.int8)
    t = np.array([[0.1, 2.4, -3.2, 6.9, -6.6, 1.3, -0.2, -0.8] * 4])
    return q, t


def _bench_flips():
    import bench
    return bench._flips


def test_rule_constant():
    assert MIDPOINT_REL == 1e-6


def test_equal_codes():
    q, t = _case()
    assert check_codes(q.copy(), q, t, packed=False) == 0.0
    assert check_codes(oracle.pack_int4(q), q, t) == 0.0
    assert _bench_flips()(q, q, t) == (0.0, 0, q.size)


@pytest.mark.parametrize("o,g,v", [
    (2, 3, 2.5),                        # exactly on the midpoint
    (2, 3, 2.5 * (1 - 0.9e-6)),         # inside the allowance, below it
    (-3, -4, -3.5 * (1 + 0.9e-6)),      # negative side
    (0, 1, 0.5 * (1 + 0.9e-6)),
    (7, 6, 6.5 * (1 - 0.9e-6)),         # the GPU rounded down
])
def test_allowed_flip(o, g, v):
    q, t = _case()
    q[0, 9], t[0, 9] = o, v
    gq = q.copy()
    gq[0, 9] = g
    assert check_codes(gq, q, t, packed=False) == pytest.approx(1 / q.size)
    assert check_codes(oracle.pack_int4(gq), q, t) == pytest.approx(1 / q.size)
    frac, outside, n = _bench_flips()(gq, q, t)
    assert (frac, outside, n) == (pytest.approx(1 / q.size), 0, q.size)


@pytest.mark.parametrize("o,g,v", [
    (2, 3, 2.5 * (1 + 1.1e-6)),         # just outside the relative allowance
    (0, 1, 0.5 - 1e-6),                 # inside 1e-6 absolutely, not relatively
    (2, 3, 2.4),                        # far from the midpoint
    (2, 4, 3.0),                        # off by two
    (2, 1, 2.5),                        # the other neighbour: midpoint 1.5
])
def test_disallowed_difference(o, g, v):
    q, t = _case()
    q[0, 9], t[0, 9] = o, v
    gq = q.copy()
    gq[0, 9] = g
    with pytest.raises(AssertionError):
        check_codes(gq, q, t, packed=False)
    with pytest.raises(AssertionError):
        check_codes(oracle.pack_int4(gq), q, t)
    assert _bench_flips()(gq, q, t)[1] == 1


def test_fraction_counts_every_allowed_flip():
    q, t = _case()
    q = np.repeat(q, 4, axis=0)
    t = np.repeat(t, 4, axis=0)
    gq = q.copy()
    for row in range(3):            # three allowed flips in 128 codes
        q[row, 1], t[row, 1] = 2, 2.5
        gq[row, 1] = 3
    assert check_codes(gq, q, t, packed=False) == pytest.approx(3 / 128)
    frac, outside, n = _bench_flips()(gq, q, t)
    assert (frac, outside, n) == (pytest.approx(3 / 128), 0, 128)
