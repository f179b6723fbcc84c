"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests retypes the oracle's formulas: each compares it with a
library routine, a closed form, a hand-derived worked example (tests/golden),
an invariant, or brute force on tiny inputs, chosen so that a plausible slip
(dropped term, wrong sign or index, transposed operand, wrong rounding) fails.
"""
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _blockdiag_h(K, b):
    """Block-diagonal normalised Sylvester Hadamard from scipy's routine."""
    hb = scipy.linalg.hadamard(b).astype(np.float64) / math.sqrt(b)
    return scipy.linalg.block_diag(*([hb] * (K // b)))


# ---------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_is_sylvester(b):
    # scipy.linalg.hadamard builds Sylvester's construction in natural order.
    h = oracle.hadamard(b)
    assert np.array_equal(h * math.sqrt(b), scipy.linalg.hadamard(b).astype(np.float64))


@pytest.mark.parametrize("b", [2, 8, 128, 256])
def test_hadamard_orthogonal(b):
    # H H^T = I: the U U^T = I requirement of CoQuant Eq. (3).
    h = oracle.hadamard(b)
    assert np.abs(h @ h.T - np.eye(b)).max() < 1e-14
    # integer form: (sqrt(b) H)(sqrt(b) H)^T = b I exactly
    hi = np.rint(h * math.sqrt(b))
    assert np.array_equal(hi @ hi.T, b * np.eye(b))


@pytest.mark.parametrize("b,K", [(4, 16), (128, 384), (256, 512), (1, 64)])
def test_rotate_equals_dense_blockdiag(b, K):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, K))
    got = oracle.rotate(x, b)
    ref = x @ _blockdiag_h(K, b)
    assert np.abs(got - ref).max() < 1e-12 * max(1.0, np.abs(ref).max())


def test_rotation_invariance_eq3():
    # (X H)(H^T W) = X W (CoQuant Eq. (3)); the weight side is rotated as rows
    # of W^T, i.e. (H^T W)^T = W^T H.
    rng = np.random.default_rng(2)
    X = rng.standard_normal((7, 256))
    Wt = rng.standard_normal((9, 256))
    for b in (2, 16, 128, 256):
        lhs = oracle.rotate(X, b) @ oracle.rotate(Wt, b).T
        rhs = X @ Wt.T
        assert np.linalg.norm(lhs - rhs) <= 1e-12 * np.linalg.norm(rhs)


def test_rotation_block_complement_eq5():
    # Splitting an orthogonal U into column blocks U = [U_l, U_h] gives
    # U_l U_l^T + U_h U_h^T = I (CoQuant Eq. (5)); the same holds for the
    # columns of the block Hadamard, probed through the oracle's rotation of
    # the identity.
    K, b = 256, 128
    U = oracle.rotate(np.eye(K), b)          # = blockdiag(H) since I H = H
    Ul, Uh = U[:, :200], U[:, 200:]
    assert np.abs(Ul @ Ul.T + Uh @ Uh.T - np.eye(K)).max() < 1e-14


# --------------------------------------------------------------- quantizer

def _read_golden(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append([c.strip() for c in line.split("|")])
    return rows


def test_worked_examples_golden():
    for name, b, xs, xhs, s, codes in _read_golden("quantizer_worked.txt"):
        b = int(b)
        x = np.array([[float(v) for v in xs.split(",")]])
        xh = np.array([float(v) for v in xhs.split(",")])
        got = oracle.rotate(x, b)[0]
        assert np.allclose(got, xh, rtol=0, atol=1e-14), name
        q, sc, _ = oracle.quantize_sym(got[None, :])
        assert abs(sc[0] - float(s)) <= 1e-15, name
        assert q[0].tolist() == [int(c) for c in codes.split(",")], name


def test_grid_values_round_trip():
    # Values already on the grid s*q (q in [-7, 7], one |q| = 7 per row) come
    # back unchanged (CoQuant Eq. (1)).  Scales are powers of two so s*q, the
    # absmax and s are exact in fp64.
    rng = np.random.default_rng(3)
    q = rng.integers(-7, 8, size=(20, 96)).astype(np.int8)
    q[np.arange(20), rng.integers(0, 96, size=20)] = rng.choice([-7, 7], size=20)
    s = 2.0 ** rng.integers(-20, 10, size=20)
    v = q.astype(np.float64) * s[:, None]
    q2, s2, t2 = oracle.quantize_sym(v)
    assert np.array_equal(q2, q)
    assert np.array_equal(s2, s)
    assert np.array_equal(t2, q.astype(np.float64))


def test_quantizer_error_bound_and_extremes():
    rng = np.random.default_rng(4)
    v = rng.standard_normal((50, 128)) * rng.uniform(0.01, 100, size=(50, 1))
    q, s, _ = oracle.quantize_sym(v)
    assert q.min() >= -7 and q.max() <= 7
    err = np.abs(v - s[:, None] * q)
    assert np.all(err <= s[:, None] / 2 * (1 + 1e-12))
    # the absmax element of each row maps to +-7 with its sign
    i = np.abs(v).argmax(axis=1)
    assert np.array_equal(q[np.arange(50), i], 7 * np.sign(v[np.arange(50), i]).astype(np.int8))
    # odd symmetry
    qn, sn, _ = oracle.quantize_sym(-v)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    # invariance of the codes under a positive power-of-two row scaling
    qs, ss, _ = oracle.quantize_sym(v * 8.0)
    assert np.array_equal(qs, q) and np.array_equal(ss, 8.0 * s)


def test_quantizer_zero_row():
    v = np.zeros((2, 64))
    v[1, 3] = -2.0
    q, s, _ = oracle.quantize_sym(v)
    assert s[0] == 0.0 and not q[0].any()
    assert s[1] == 2.0 / 7.0 and q[1, 3] == -7 and np.count_nonzero(q[1]) == 1


def test_quantizer_ties_to_even():
    # v/s lands exactly on k + 1/2 (amax 7, s = 1): half-to-even.
    v = np.array([[7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 6.5]])
    q, s, _ = oracle.quantize_sym(v)
    assert q[0].tolist() == [7, 0, 2, 2, 0, -2, -2, 6]


# ------------------------------------------------------------- int4 layout

def test_pack_golden():
    rows = dict((r[0], r[1]) for r in _read_golden("pack_int4.txt"))
    codes = np.array([[int(c) for c in rows["codes"].split(",")]], dtype=np.int8)
    want = np.array([[int(b, 16) for b in rows["bytes"].split(",")]], dtype=np.uint8)
    assert np.array_equal(oracle.pack_int4(codes), want)
    assert np.array_equal(oracle.unpack_int4(want), codes)


def test_pack_round_trip():
    rng = np.random.default_rng(5)
    q = rng.integers(-7, 8, size=(9, 256)).astype(np.int8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(q)), q)


# ------------------------------------------------------------ integer GEMM

def test_int_gemm_bruteforce():
    rng = np.random.default_rng(6)
    for (M, N, K) in [(1, 1, 128), (3, 5, 128), (8, 8, 256)]:
        a = rng.integers(-7, 8, size=(M, K)).astype(np.int8)
        b = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
        acc = oracle.int_gemm(a, b)
        for m in range(M):
            for n in range(N):
                want = 0
                for k in range(K):
                    want += int(a[m, k]) * int(b[n, k])
                assert acc[m, n] == want


def test_int_gemm_accumulator_bound():
    # |acc| <= 49 K fits INT32 even at K = 28672 (TwinQuant notes, Figure 4:
    # INT32 accumulation avoids overflow).
    K = 28672
    a = np.full((1, K), 7, dtype=np.int8)
    b = np.full((2, K), -7, dtype=np.int8)
    b[1] = 7
    acc = oracle.int_gemm(a, b)
    assert acc[0, 0] == -49 * K and acc[0, 1] == 49 * K
    assert 49 * K < 2 ** 31 - 1


# -------------------------------------------------------------- bf16 / LR

def test_round_bf16_matches_torch():
    # torch rounds fp32 -> bf16 to nearest even; feed fp32-representable values
    # so a single rounding is compared, including exact bf16 ties.
    rng = np.random.default_rng(7)
    x32 = (rng.standard_normal(4000) * 10.0 ** rng.uniform(-30, 30, 4000)).astype(np.float32)
    ties = (np.float32(1.0) + np.float32(2.0 ** -8) * np.arange(1, 40, 2, dtype=np.float32))
    x32 = np.concatenate([x32, ties, -ties, np.float32([0.0, 1e-40, -3e38, 3.3e38])])
    want = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    got = oracle.round_bf16(x32.astype(np.float64))
    assert np.array_equal(got, want)


def test_lowrank_matches_matmul():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((6, 256))
    L1t = rng.standard_normal((16, 256)) * 0.05
    L2t = rng.standard_normal((64, 16)) * 0.05
    XL1, lr = oracle.lowrank(X, L1t, L2t, round_mid=False)
    assert np.abs(XL1 - X @ L1t.T).max() < 1e-12
    assert np.abs(lr - XL1 @ L2t.T).max() < 1e-12
    _, lr_r = oracle.lowrank(X, L1t, L2t, round_mid=True)
    want = oracle.round_bf16(XL1) @ L2t.T
    assert np.abs(lr_r - want).max() < 1e-12


# ---------------------------------------------------------- layer reductions

def test_rank0_is_plain_quantized_matmul():
    sh = synth.CONFIGS["tiny"].with_(r=0, M=5)
    L = synth.make_layer(sh)
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], sh.had_block)
    # dequant(Q4(X H) Q4(H^T W)): recompute the product of dequantized codes
    # with numpy's matmul from the oracle's codes and scales.
    deq = (o["qx"] * o["s_x"][:, None]) @ (o["qw"] * o["s_w"][:, None]).T
    assert np.abs(o["Y64"] - deq).max() <= 1e-12 * np.abs(deq).max()
    assert not np.any(o["lr"])


def test_exact_lowrank_weight_reduces_to_xl1l2():
    # R = 0 (W exactly rank r): the residual codes vanish and Y = bf16(X L1) L2.
    sh = synth.CONFIGS["tiny"].with_(M=4)
    L = synth.make_layer(sh)
    Rt = torch.zeros_like(L["Rt"])
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], Rt, sh.had_block)
    assert not o["qw"].any() and not o["s_w"].any()
    X = L["X"].double().numpy()
    xl1 = torch.from_numpy(X @ L["L1t"].double().numpy().T).float().to(torch.bfloat16).double().numpy()
    want = xl1 @ L["L2t"].double().numpy().T
    assert np.abs(o["Y64"] - want).max() <= 1e-6 * np.abs(want).max()


def test_layer_approximates_xw_and_rotation_helps():
    # Plausibility (CoQuant Eqs. (10)-(12), AQNM): the W4A4 layer is close to
    # the exact X W, and the Hadamard rotation lowers the error on inputs with
    # outlier channels (CoQuant section 3, "Hadamard-based transform").
    sh = synth.CONFIGS["tiny"].with_(M=64)
    L = synth.make_layer(sh)
    X = L["X"].double().numpy()
    W = L["Rt"].double().numpy().T + L["L1t"].double().numpy().T @ L["L2t"].double().numpy().T
    ref = X @ W
    errs = {}
    for b in (1, 256):
        o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b)
        errs[b] = np.linalg.norm(o["Y64"] - ref) / np.linalg.norm(ref)
    assert errs[256] < 0.25
    assert errs[256] < 0.7 * errs[1]
