"""Comparison rules shared by the parity tests (test-side only)."""
from __future__ import annotations

import numpy as np

import oracle

# Output tolerance of the layer (bf16 Y against the oracle's fp64 Y):
# relative Frobenius error and max-abs error relative to max|Y|.
Y_REL_FRO = 2e-3
Y_MAX_ABS = 1e-2
# Codes may differ by one only where the oracle's value v/s lies within this
# relative distance of the rounding midpoint between the two codes.
MIDPOINT_REL = 1e-6


def check_codes(gpu_packed, orc_q, orc_t, what="codes", packed=True):
    """Unpack the GPU's packed codes (or take them one per byte when
    packed=False) and compare them with the oracle's.

    Returns the fraction of codes that differ (all of them allowed midpoint
    flips); raises AssertionError on any other difference.
    """
    if packed:
        gq = oracle.unpack_int4(np.ascontiguousarray(gpu_packed))
    else:
        gq = np.asarray(gpu_packed).astype(np.int8)
    assert gq.shape == orc_q.shape, (gq.shape, orc_q.shape)
    diff = gq.astype(np.int32) - orc_q.astype(np.int32)
    bad = diff != 0
    if not bad.any():
        return 0.0
    idx = np.nonzero(bad)
    d = diff[idx]
    t = orc_t[idx]
    mid = (gq[idx].astype(np.float64) + orc_q[idx].astype(np.float64)) / 2.0
    ok = (np.abs(d) == 1) & (np.abs(t - mid) <= MIDPOINT_REL * np.abs(t))
    if not ok.all():
        j = np.nonzero(~ok)[0][:5]
        raise AssertionError(
            f"{what}: {int((~ok).sum())} codes differ outside the midpoint allowance; "
            f"e.g. at {[tuple(int(a[i]) for a in idx) for i in j]}: gpu {gq[idx][j]} "
            f"oracle {orc_q[idx][j]} v/s {t[j]}")
    return float(bad.sum()) / bad.size


def check_scales(gpu, orc, what="scales", rel=2e-6):
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - orc)
    lim = rel * np.abs(orc)
    assert np.all(err <= lim), f"{what}: max rel err {np.max(err / np.maximum(np.abs(orc), 1e-300))}"


def check_xl1(gpu, X, L1t, orc_xl1, rel=1e-5):
    """|gpu - oracle| <= rel * sum_k |X[m,k] L1[k,j]| elementwise."""
    gpu = np.asarray(gpu, dtype=np.float64)
    bound = np.abs(X) @ np.abs(L1t).T
    err = np.abs(gpu - orc_xl1)
    assert np.all(err <= rel * bound + 1e-30), \
        f"XL1: worst err/bound {np.max(err / np.maximum(bound, 1e-300))}"


def check_y(gpu_y, y64, what="Y"):
    gpu_y = np.asarray(gpu_y, dtype=np.float64)
    fro = np.linalg.norm(gpu_y - y64) / max(np.linalg.norm(y64), 1e-300)
    mx = np.abs(gpu_y - y64).max() / max(np.abs(y64).max(), 1e-300)
    assert fro <= Y_REL_FRO, f"{what}: relative Frobenius error {fro:.3e} > {Y_REL_FRO}"
    assert mx <= Y_MAX_ABS, f"{what}: max-abs error {mx:.3e} of max|Y| > {Y_MAX_ABS}"
    return fro, mx


def y_reference(gpu_codes, o, flips, gpu_wcodes=None, wflips=0):
    """The reference for Y: the oracle's fp64 Y64 when the GPU's codes equal
    the oracle's (flips == wflips == 0), else the oracle's epilogue on the
    GPU's activation codes (if they hold flips) and weight codes (if those
    do).  The second case is only reached after check_codes has shown that
    every difference is an allowed midpoint flip: one flip moves a token's
    whole row (or a channel's whole column) of Y by s_x s_w q, which the
    output tolerance is not meant to absorb (it can reach 2e-3 relative
    Frobenius alone)."""
    if flips == 0 and wflips == 0:
        return o["Y64"]
    qa = np.asarray(gpu_codes).astype(np.int8) if flips else o["qx"]
    qw = np.asarray(gpu_wcodes).astype(np.int8) if wflips else o["qw"]
    return oracle.epilogue(o["s_x"], o["s_w"], oracle.int_gemm(qa, qw), o["lr"])


def y_given_codes(gpu_codes, o):
    """The oracle's epilogue evaluated on the GPU's activation codes (already
    checked by check_codes to differ from the oracle's only by midpoint
    flips) with the oracle's scales, weight codes and low-rank term: the
    reference for Y when the codes may legitimately differ."""
    acc = oracle.int_gemm(np.asarray(gpu_codes).astype(np.int8), o["qw"])
    return oracle.epilogue(o["s_x"], o["s_w"], acc, o["lr"])
