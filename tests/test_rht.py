"""Randomized Hadamard transform (the TORQUE page's randomized Hadamard
abstract: random signs, then the Hadamard): the rotation becomes D H with D
a +-1 diagonal given as a bit mask.  CPU pins of the oracle's signed
rotation, then (gpu) the library's signed entry points against it."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_scales, check_y, y_reference

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rht_worked.txt")


def _rng_signs(K, seed):
    words = np.random.default_rng(seed).integers(0, 2 ** 32, size=K // 32, dtype=np.uint64)
    return words.astype(np.uint32)


def _blockdiag_h(K, b):
    h = oracle.hadamard(b)
    out = np.zeros((K, K))
    for i in range(0, K, b):
        out[i:i + b, i:i + b] = h
    return out


# ------------------------------------------------------------------ CPU pins

def test_hand_worked_examples():
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        name, b, mask, x, xdh, s, codes = [f.strip() for f in line.split("|")]
        b = int(b)
        x = np.array([float(v) for v in x.split(",")])[None, :]
        d = oracle.signs_from_bits(np.array([int(mask, 16)], dtype=np.uint32), x.shape[1])
        got = oracle.rotate(x, b, d)
        assert np.allclose(got, [float(v) for v in xdh.split(",")], rtol=0, atol=1e-15), name
        q, sc, _ = oracle.quantize_sym(got)
        assert sc[0] == pytest.approx(float(s), rel=1e-15), name
        assert list(q[0]) == [int(v) for v in codes.split(",")], name


def test_mask_bit_order():
    # words [0x0000000B, 0x80000000]: columns 0, 1, 3 and 63 negated
    d = oracle.signs_from_bits(np.array([0xB, 0x80000000], dtype=np.uint32), 64)
    assert sorted(np.nonzero(d < 0)[0].tolist()) == [0, 1, 3, 63]
    assert set(d.tolist()) == {1.0, -1.0}


@pytest.mark.parametrize("b", [2, 16, 128, 256])
def test_signed_rotation_is_orthogonal(b):
    K = 512
    d = oracle.signs_from_bits(_rng_signs(K, b), K)
    U = oracle.rotate(np.eye(K), b, d)        # the matrix D H itself
    assert np.abs(U @ U.T - np.eye(K)).max() < 1e-13


@pytest.mark.parametrize("b", [4, 128])
def test_signs_come_before_the_hadamard(b):
    """A unit row e_k maps to d_k times row k of H (x D H); applying the
    signs after H instead would give row k of H times D."""
    K = 256
    d = oracle.signs_from_bits(_rng_signs(K, 7), K)
    H = _blockdiag_h(K, b)
    E = oracle.rotate(np.eye(K), b, d)
    assert np.allclose(E, d[:, None] * H, rtol=0, atol=1e-15)
    assert not np.allclose(E, H * d[None, :])


def test_eq3_invariance_with_signs():
    """CoQuant Eq. (3) with U = D H: (X D H)((D H)^T W) = X W."""
    K, M, N, b = 512, 9, 40, 128
    rng = np.random.default_rng(3)
    X, W = rng.normal(size=(M, K)), rng.normal(size=(K, N))
    d = oracle.signs_from_bits(_rng_signs(K, 11), K)
    lhs = oracle.rotate(X, b, d) @ oracle.rotate(W.T, b, d).T
    assert np.abs(lhs - X @ W).max() <= 1e-12 * np.abs(X @ W).max()


def test_all_plus_and_all_minus_signs():
    K, b = 256, 64
    X = np.random.default_rng(5).normal(size=(6, K))
    plus = oracle.signs_from_bits(np.zeros(K // 32, dtype=np.uint32), K)
    minus = oracle.signs_from_bits(np.full(K // 32, 0xFFFFFFFF, dtype=np.uint32), K)
    assert np.array_equal(oracle.rotate(X, b, plus), oracle.rotate(X, b))
    assert np.array_equal(oracle.rotate(X, b, minus), -oracle.rotate(X, b))
    qp, sp, _ = oracle.quantize_sym(oracle.rotate(X, b))
    qm, sm, _ = oracle.quantize_sym(oracle.rotate(X, b, minus))
    assert np.array_equal(qm, -qp) and np.array_equal(sm, sp)


def test_signed_layer_is_a_plausible_approximation():
    """The layer with D H on both sides approximates X W about as well as
    with H alone (the signs only re-mix the Hadamard blocks)."""
    sh = synth.CONFIGS["decode"].with_(M=32, K=1024, N=256, r=32)
    L = synth.make_layer(sh, seed=2)
    d = oracle.signs_from_bits(_rng_signs(1024, 13), 1024)
    W = L["Rt"].double().numpy().T + L["L1t"].double().numpy().T @ L["L2t"].double().numpy().T
    exact = L["X"].double().numpy() @ W
    e_plain = np.linalg.norm(oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], 128)["Y64"] - exact)
    e_rht = np.linalg.norm(oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], 128, signs=d)["Y64"] - exact)
    assert e_rht < 1.5 * e_plain and e_plain < 1.5 * e_rht
    assert e_rht < 0.2 * np.linalg.norm(exact)   # the plain layer is at ~11 % (4-bit codes)


# ---------------------------------------------------------------- the GPU

@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


def _dev_signs(K, seed):
    return torch.from_numpy(_rng_signs(K, seed).view(np.int32)).cuda()


@pytest.mark.gpu
@pytest.mark.parametrize("b", [128, 256])
def test_signed_weight_pack_matches_oracle(tq, b):
    sh = synth.CONFIGS["decode"].with_(M=4, K=2048, N=384, r=0, had_block=b)
    L = synth.make_layer(sh, seed=21)
    sg = _dev_signs(2048, 99 + b)
    d = oracle.signs_from_bits(sg.cpu().numpy().view(np.uint32), 2048)
    Wq, s_w = tq.tq_pack_weight_rht(L["Rt"].cuda(), b, sg)
    torch.cuda.synchronize()
    w = oracle.pack_weight(L["Rt"], b, signs=d)
    check_codes(Wq.cpu().numpy(), w["qw"], w["t_w"], "signed weight codes")
    check_scales(s_w.cpu().numpy(), w["s_w"], "signed s_w")


@pytest.mark.gpu
# M >= 64 with b <= 128 runs the tensor-core activation kernel, which negates
# the masked columns of each staged X block (and of L1^T) in shared memory;
# r = 160 adds an X-L1-only launch (unmasked); the rest run the butterflies
@pytest.mark.parametrize("M,b,r", [(1, 128, 32), (16, 256, 16), (200, 128, 64), (70, 256, 0),
                                   (300, 64, 16), (1000, 128, 128), (520, 128, 160),
                                   (130, 32, 0)])
def test_signed_activation_codes_match_oracle(tq, M, b, r):
    from tests.parity_util import check_xl1
    K = 4096
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=256, r=r, had_block=b)
    L = synth.make_layer(sh, seed=22)
    sg = _dev_signs(K, 7 * M + b)
    d = oracle.signs_from_bits(sg.cpu().numpy().view(np.uint32), K)
    Xq, s_x, XL1 = tq.tq_quantize_act_rht(L["X"].cuda(), b, sg, L["L1t"].cuda() if r else None)
    torch.cuda.synchronize()
    a = oracle.quantize_act(L["X"], b, L["L1t"] if r else None, signs=d)
    fx = check_codes(Xq.cpu().numpy(), a["qx"], a["t_x"], "signed activation codes")
    check_scales(s_x.cpu().numpy(), a["s_x"], "signed s_x")
    if r:   # X L1 reads the unrotated X: unchanged by the signs
        check_xl1(XL1.cpu().numpy(), L["X"].double().numpy(), L["L1t"].double().numpy(), a["XL1"])
    print(f"FLIPS rht act M={M} b={b}: x={fx:.3e}")


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,N,r,b", [(16, 4096, 4096, 32, 128), (1, 4096, 1024, 16, 256),
                                       (5, 1024, 520, 32, 64), (200, 2048, 512, 64, 128),
                                       (600, 4096, 1024, 32, 128), (130, 1024, 264, 16, 256)])
def test_signed_layer_matches_oracle(tq, M, K, N, r, b):
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, seed=23, device="cuda" if K * N >= 1 << 22 else "cpu")
    sg = _dev_signs(K, M + K + b)
    d = oracle.signs_from_bits(sg.cpu().numpy().view(np.uint32), K)
    Wq, s_w = tq.tq_pack_weight_rht(L["Rt"].cuda(), b, sg)
    Y = tq.tq_w4a4_lr_layer_rht(L["X"].cuda(), sg, L["L1t"].cuda(), Wq, s_w, L["L2t"].cuda(), b)
    Xq, _, _ = tq.tq_quantize_act_rht(L["X"].cuda(), b, sg)
    torch.cuda.synchronize()
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b, signs=d)
    q = oracle.unpack_int4(Xq.cpu().numpy())
    qw = oracle.unpack_int4(Wq.cpu().numpy())
    fx = check_codes(q, o["qx"], o["t_x"], "signed codes", packed=False)
    fw = check_codes(qw, o["qw"], o["t_w"], "signed weight codes", packed=False)
    fro, mx = check_y(Y.double().cpu().numpy(), y_reference(q, o, fx, qw, fw),
                      f"signed layer M={M} K={K} N={N}")
    print(f"FLIPS rht layer M={M} path={tq.tq_layer_path(M, N, K, r, b)}: fro={fro:.3e}")


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,N,b", [(300, 1024, 384, 128), (1000, 4096, 1024, 64)])
def test_signed_layer_int8_path_equals_packed_path_at_rank0(tq, M, K, N, b):
    # above 128 tokens the signed layer writes one code per byte from the
    # tensor-core activation kernel and runs the int8-code GEMM; at rank 0
    # its Y equals the packed codes of the same kernel through the packed-code
    # GEMM bit for bit (same codes, exact integer sums, the same fp32 epilogue)
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=0, had_block=b)
    L = synth.make_layer(sh, seed=25, device="cuda")
    sg = _dev_signs(K, M + 7)
    X = L["X"].cuda()
    Wq, s_w = tq.tq_pack_weight_rht(L["Rt"].cuda(), b, sg)
    assert tq.tq_layer_path(M, N, K, 0, b) == "codes_i8"
    Y = tq.tq_w4a4_lr_layer_rht(X, sg, None, Wq, s_w, None, b)
    Xq, s_x, _ = tq.tq_quantize_act_rht(X, b, sg)
    Y2 = tq.tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


@pytest.mark.gpu
@pytest.mark.parametrize("M,r", [(300, 64), (700, 160)])
def test_masked_tensor_core_kernel_against_the_plain_one(tq, M, r):
    # the tensor-core activation kernel with a sign mask: an all-zero mask
    # gives the plain kernel's outputs bit for bit, and with any mask X L1
    # is unchanged bit for bit ((x D)(D L1) = x L1 with exact sign flips and
    # the same summation order); the codes of a mask equal those of the plain
    # kernel on X with its masked columns negated (the same products summed
    # in the same order)
    K, b = 2048, 128
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=256, r=r, had_block=b)
    L = synth.make_layer(sh, seed=26, device="cuda")
    X, L1t = L["X"].cuda(), L["L1t"].cuda()
    zero = torch.zeros(K // 32, dtype=torch.int32, device="cuda")
    sg = _dev_signs(K, M + 3)
    d = torch.from_numpy(oracle.signs_from_bits(sg.cpu().numpy().view(np.uint32), K)).cuda()
    plain = tq.tq_quantize_act(X, b, L1t)
    masked0 = tq.tq_quantize_act_rht(X, b, zero, L1t)
    masked = tq.tq_quantize_act_rht(X, b, sg, L1t)
    negated = tq.tq_quantize_act((X.double() * d).to(torch.bfloat16), b, L1t)
    torch.cuda.synchronize()
    assert all(torch.equal(u, v) for u, v in zip(plain, masked0))
    assert torch.equal(masked[2], plain[2])
    assert torch.equal(masked[0], negated[0]) and torch.equal(masked[1], negated[1])


@pytest.mark.gpu
def test_zero_mask_equals_the_plain_calls(tq):
    sh = synth.CONFIGS["decode"].with_(M=16, K=4096, N=1024, r=32)
    L = synth.make_layer(sh, seed=24, device="cuda")
    zero = torch.zeros(4096 // 32, dtype=torch.int32, device="cuda")
    X, L1t, L2t, Rt = (L[k].cuda() for k in ("X", "L1t", "L2t", "Rt"))
    Wq, s_w = tq.tq_pack_weight(Rt, 128)
    Wq_r, s_w_r = tq.tq_pack_weight_rht(Rt, 128, zero)
    a, b = tq.tq_quantize_act(X, 128, L1t), tq.tq_quantize_act_rht(X, 128, zero, L1t)
    Y = tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128)
    Y_r = tq.tq_w4a4_lr_layer_rht(X, zero, L1t, Wq, s_w, L2t, 128)
    torch.cuda.synchronize()
    assert torch.equal(Wq, Wq_r) and torch.equal(s_w, s_w_r)
    assert all(torch.equal(u, v) for u, v in zip(a, b))
    assert torch.equal(Y, Y_r)


def test_signed_entry_argument_checks():
    import ctypes

    import rank_int4_gemm_b200 as tq
    lib = tq.tq.raw()
    P = ctypes.c_void_p
    F = 0x1000
    assert lib.tq_pack_weight_rht(P(F), 8, 256, 128, None, P(F), P(F), None) == 1     # no mask
    assert lib.tq_pack_weight_rht(P(F), 8, 256, 128, P(F + 4), P(F), P(F), None) == 3
    assert lib.tq_quantize_act_rht(P(F), 4, 256, 128, None, None, 0, P(F), P(F), None, None) == 1
    assert lib.tq_w4a4_lr_layer_rht(P(F), None, None, P(F), P(F), None, 4, 64, 256, 0, 128, P(F),
                                    P(F), ctypes.c_size_t(1 << 20), None) == 1


# ------------------------------------------ composed randomized Hadamards

def _mask(sgn):
    return np.array([1.0 if c == "+" else -1.0 for c in sgn])


def test_composed_hand_worked_examples():
    path = os.path.join(os.path.dirname(__file__), "golden", "rht_composed_worked.txt")
    for line in open(path).read().splitlines():
        if line.startswith("#") or not line.strip():
            continue
        name, b, masks, x, want = [f.strip() for f in line.split("|")]
        d = np.stack([_mask(m) for m in masks.split(";")])
        x = np.array([float(v) for v in x.split(",")])[None, :]
        got = oracle.rotate(x, int(b), signs=d)[0]
        assert np.allclose(got, [float(v) for v in want.split(",")], rtol=0, atol=1e-14), name


@pytest.mark.parametrize("b,n", [(2, 2), (16, 3), (128, 2)])
def test_composed_rotation_is_the_product_of_single_transforms(b, n):
    # against matrices built here from scipy's Hadamard: D_1 Hd D_2 Hd ...
    from scipy.linalg import hadamard
    K = 4 * b
    rng = np.random.default_rng(b + n)
    d = rng.choice([-1.0, 1.0], size=(n, K))
    Hd = np.kron(np.eye(K // b), hadamard(b) / np.sqrt(b))
    Q = np.eye(K)
    for i in range(n):
        Q = Q @ np.diag(d[i]) @ Hd
    x = rng.normal(size=(5, K))
    assert np.allclose(oracle.rotate(x, b, signs=d), x @ Q, rtol=0, atol=1e-12)
    assert np.allclose(Q @ Q.T, np.eye(K), atol=1e-12)  # orthogonal
    # the single-transform case of the same call
    assert np.allclose(oracle.rotate(x, b, signs=d[:1]), oracle.rotate(x, b, signs=d[0]),
                       rtol=0, atol=0)


@pytest.mark.parametrize("b", [4, 128])
def test_two_all_plus_masks_give_the_identity(b):
    x = np.random.default_rng(b).normal(size=(3, 2 * b))
    assert np.allclose(oracle.rotate(x, b, signs=np.ones((2, 2 * b))), x, rtol=0, atol=1e-12)


def test_composed_eq3_invariance_and_bit_masks():
    # (X Q)(Q^T W) = X W for the composed transform on both sides; masks as
    # bit words decode row by row
    rng = np.random.default_rng(7)
    K, b = 256, 64
    bits = rng.integers(0, 2**32, size=(3, K // 32), dtype=np.uint64).astype(np.uint32)
    d = oracle.signs_from_bits(bits, K)
    assert d.shape == (3, K)
    for i in range(3):
        assert np.array_equal(d[i], oracle.signs_from_bits(bits[i], K))
    X, W = rng.normal(size=(4, K)), rng.normal(size=(6, K))
    lhs = oracle.rotate(X, b, signs=d) @ oracle.rotate(W, b, signs=d).T
    assert np.allclose(lhs, X @ W.T, rtol=0, atol=1e-10)


def _dev_masks(n, K, seed):
    return torch.stack([_dev_signs(K, seed + 101 * i) for i in range(n)]).contiguous()


@pytest.mark.gpu
@pytest.mark.parametrize("n,b", [(2, 128), (3, 256), (2, 16)])
def test_composed_weight_and_activation_codes_match_oracle(tq, n, b):
    K, M = 2048, 200
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=384, r=32, had_block=b)
    L = synth.make_layer(sh, seed=31)
    sg = _dev_masks(n, K, 5 * b + n)
    d = oracle.signs_from_bits(sg.cpu().numpy().view(np.uint32), K)
    assert d.shape == (n, K)
    Wq, s_w = tq.tq_pack_weight_rht(L["Rt"].cuda(), b, sg)
    Xq, s_x, _ = tq.tq_quantize_act_rht(L["X"].cuda(), b, sg)
    torch.cuda.synchronize()
    w = oracle.pack_weight(L["Rt"], b, signs=d)
    check_codes(Wq.cpu().numpy(), w["qw"], w["t_w"], f"composed ({n}) weight codes")
    check_scales(s_w.cpu().numpy(), w["s_w"], f"composed ({n}) s_w")
    a = oracle.quantize_act(L["X"], b, signs=d)
    fx = check_codes(Xq.cpu().numpy(), a["qx"], a["t_x"], f"composed ({n}) activation codes")
    check_scales(s_x.cpu().numpy(), a["s_x"], f"composed ({n}) s_x")
    print(f"FLIPS rht{n} act b={b}: x={fx:.3e}")


@pytest.mark.gpu
@pytest.mark.parametrize("n,M,K,N,r,b", [(2, 16, 4096, 4096, 32, 128), (3, 1, 2048, 1024, 64, 256),
                                         (2, 300, 2048, 512, 32, 128), (2, 40, 1024, 264, 16, 64)])
def test_composed_layer_matches_oracle(tq, n, M, K, N, r, b):
    # the fused decode kernel (M <= 16), the int8-code path (M > 128) and the
    # packed path (in between) with n composed transforms on both sides
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, seed=33, device="cuda" if K * N >= 1 << 22 else "cpu")
    sg = _dev_masks(n, K, M + K + n)
    d = oracle.signs_from_bits(sg.cpu().numpy().view(np.uint32), K)
    Wq, s_w = tq.tq_pack_weight_rht(L["Rt"].cuda(), b, sg)
    Y = tq.tq_w4a4_lr_layer_rht(L["X"].cuda(), sg, L["L1t"].cuda(), Wq, s_w, L["L2t"].cuda(), b)
    Xq, _, _ = tq.tq_quantize_act_rht(L["X"].cuda(), b, sg)
    torch.cuda.synchronize()
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b, signs=d)
    q = oracle.unpack_int4(Xq.cpu().numpy())
    qw = oracle.unpack_int4(Wq.cpu().numpy())
    fx = check_codes(q, o["qx"], o["t_x"], "composed codes", packed=False)
    fw = check_codes(qw, o["qw"], o["t_w"], "composed weight codes", packed=False)
    fro, mx = check_y(Y.double().cpu().numpy(), y_reference(q, o, fx, qw, fw),
                      f"composed ({n}) layer M={M} K={K} N={N}")
    print(f"FLIPS rht{n} layer M={M} path={tq.tq_layer_path(M, N, K, r, b)}: fro={fro:.3e}")


def test_composed_entry_argument_checks():
    import ctypes

    import rank_int4_gemm_b200 as tq
    lib = tq.tq.raw()
    P = ctypes.c_void_p
    F = 0x1000
    # n_rht outside 1..3
    for n in (0, 4):
        assert lib.tq_pack_weight_rhtn(P(F), 8, 256, 128, P(F), n, P(F), P(F), None) == 1
        assert lib.tq_w4a4_lr_layer_rhtn(P(F), P(F), n, None, P(F), P(F), None, 16, 256, 256, 0,
                                         128, P(F), P(F), ctypes.c_size_t(1 << 20), None) == 1
