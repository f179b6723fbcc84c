"""The comparison rules every parity claim rests on, pinned on hand-made
cases (host only).

Codes: a GPU code may differ from the oracle's only by one, and only where
the oracle's v/s lies within 1e-6 relative of the midpoint between the two
codes (round to nearest, CoQuant Eq. (1); the allowance covers the fp32
summation order of the rotation).  Both the tests' checker and the
benchmark's flip counter follow it; a checker that measured the distance
absolutely, to the wrong midpoint, or let differences of two through would
fail here.

Y: relative Frobenius error <= 2e-3 and max-abs error <= 1e-2 max|Y|
against the oracle's fp64 Y, the reference being the oracle's epilogue on
the GPU's codes where those hold allowed flips.  X L1: elementwise within
1e-5 sum_k |X L1| (fp32 accumulation of bf16 products)."""
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


# ------------------------------------------------------------------- Y, X L1

from tests.parity_util import Y_MAX_ABS, Y_REL_FRO, check_xl1, check_y, y_reference  # noqa: E402


def test_y_tolerances():
    assert (Y_REL_FRO, Y_MAX_ABS) == (2e-3, 1e-2)
    rng = np.random.default_rng(1)
    y = rng.normal(size=(64, 48))
    assert check_y(y.copy(), y) == (0.0, 0.0)
    fro, mx = check_y(y * (1 + 1.9e-3), y)
    assert fro == pytest.approx(1.9e-3) and mx <= 1.9e-3
    with pytest.raises(AssertionError):
        check_y(y * (1 + 2.1e-3), y)           # Frobenius just over
    z = y.copy()
    z[5, 7] += 1.1e-2 * np.abs(y).max()       # one element over the max-abs bound
    assert np.linalg.norm(z - y) / np.linalg.norm(y) < Y_REL_FRO
    with pytest.raises(AssertionError):
        check_y(z, y)


def test_xl1_bound_is_relative_to_the_absolute_products():
    rng = np.random.default_rng(2)
    X = rng.normal(size=(3, 64))
    L1t = rng.normal(size=(4, 64))
    exact = X @ L1t.T
    bound = np.abs(X) @ np.abs(L1t).T
    check_xl1(exact + 0.9e-5 * bound, X, L1t, exact)
    with pytest.raises(AssertionError):
        check_xl1(exact + 1.1e-5 * bound * (np.arange(12).reshape(3, 4) == 5), X, L1t, exact)


def test_y_reference_follows_the_gpu_codes_only_where_they_flip():
    # two tokens, 32 columns, two channels; the GPU's activation code of
    # token 0, column 3 differs by one (an allowed flip): the reference moves
    # by s_x[0] s_w[n] qw[n][3] in row 0 only
    rng = np.random.default_rng(3)
    qx = rng.integers(-7, 8, size=(2, 32)).astype(np.int8)
    qw = rng.integers(-7, 8, size=(2, 32)).astype(np.int8)
    s_x, s_w = np.array([0.5, 0.25]), np.array([0.125, 2.0])
    lr = rng.normal(size=(2, 2))
    o = {"qx": qx, "qw": qw, "s_x": s_x, "s_w": s_w, "lr": lr, "Y64": object()}
    assert y_reference(qx, o, 0) is o["Y64"]
    g = qx.copy()
    g[0, 3] += 1 if g[0, 3] < 7 else -1
    ref = y_reference(g, o, 1 / 64)
    for m in range(2):
        for n in range(2):
            acc = sum(int(g[m, k]) * int(qw[n, k]) for k in range(32))
            assert ref[m, n] == pytest.approx(s_x[m] * s_w[n] * acc + lr[m, n], rel=1e-14)
    # and the weight codes likewise, with the oracle's activation codes
    gw = qw.copy()
    gw[1, 0] = -gw[1, 0] if gw[1, 0] else 1
    ref = y_reference(qx, o, 0, gw, 1 / 64)
    for m in range(2):
        acc = sum(int(qx[m, k]) * int(gw[1, k]) for k in range(32))
        assert ref[m, 1] == pytest.approx(s_x[m] * s_w[1] * acc + lr[m, 1], rel=1e-14)
