"""Per-token asymmetric activation codes (CoQuant Eq. (1) with a zero-point,
chosen from the row's range): the oracle pinned on CPU, then
tq_quantize_act_asym_i8 + tq_weight_code_sums + tq_w4a4_lr_gemm_a8_asym
against it."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_y


# ------------------------------------------------------------ oracle pins

def test_asym_grid_values_round_trip():
    rng = np.random.default_rng(1)
    z, s = -3.25, 0.125  # dyadic: z + s q is exact in fp64
    q = rng.integers(0, 16, size=(5, 64))
    q[:, 0], q[:, 1] = 0, 15  # the row's min and max are on the grid ends
    x = z + s * q
    gq, gs, gz, t = oracle.quantize_asym(x)
    assert np.array_equal(gq, q)
    assert np.all(gs == s) and np.all(gz == z)
    assert np.array_equal(t, q.astype(np.float64))


def test_asym_error_bound_ends_and_invariances():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(8, 256)) * 3 + 1.5
    q, s, z, _ = oracle.quantize_asym(x)
    assert q.min() == 0 and q.max() == 15
    assert np.all(np.abs(x - (s[:, None] * q + z[:, None])) <= s[:, None] / 2 * (1 + 1e-12))
    lo, hi = x.argmin(axis=1), x.argmax(axis=1)
    assert np.all(q[np.arange(8), lo] == 0) and np.all(q[np.arange(8), hi] == 15)
    # a dyadic shift moves only the zero-point; doubling moves only the scale
    q2, s2, z2, _ = oracle.quantize_asym(x + 0.5)
    assert np.array_equal(q2, q) and np.allclose(z2, z + 0.5, rtol=0, atol=1e-12) and np.allclose(s2, s)
    q3, s3, z3, _ = oracle.quantize_asym(2 * x)
    assert np.array_equal(q3, q) and np.array_equal(s3, 2 * s) and np.array_equal(z3, 2 * z)


def test_asym_constant_row():
    q, s, z, _ = oracle.quantize_asym(np.full((2, 32), -0.75))
    assert np.all(q == 0) and np.all(s == 0) and np.all(z == -0.75)


def test_asym_layer_is_the_dequantized_product():
    """layer_asym against dequantize-then-multiply written out on a tiny layer."""
    sh = synth.CONFIGS["tiny"].with_(M=5, K=64, N=24, r=8, had_block=32)
    L = synth.make_layer(sh, seed=4)
    o = oracle.layer_asym(L["X"], L["L1t"], L["L2t"], L["Rt"], 32)
    Xh = oracle.rotate(L["X"], 32)
    q, s, z, _ = oracle.quantize_asym(Xh)
    Xhat = s[:, None] * q + z[:, None]
    w = oracle.pack_weight(L["Rt"], 32)
    What = w["s_w"][:, None] * w["qw"]
    _, lr = oracle.lowrank(L["X"], L["L1t"], L["L2t"])
    want = Xhat @ What.T + lr
    assert np.allclose(o["Y64"], want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


# ---------------------------------------------------------------- the GPU

@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


CASES = [
    # name, M, K, N, r, b, offset added to X (a row mean the zero-point absorbs)
    ("tiles", 300, 1024, 256, 32, 128, 0.0),
    ("offset_rows", 200, 512, 136, 16, 128, 2.0),
    ("one_token", 1, 512, 128, 16, 64, 0.0),
    ("rank0_block16", 130, 768, 64, 0, 16, -1.0),
    ("no_rotation", 150, 256, 128, 32, 1, 0.5),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,K,N,r,b,off", CASES, ids=[c[0] for c in CASES])
def test_asym_path_matches_oracle(tq, name, M, K, N, r, b, off):
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, seed=7)
    X = (L["X"].float() + off).to(torch.bfloat16)
    dev = lambda t: t.cuda() if r else None  # noqa: E731
    Wq, s_w = tq.tq_pack_weight(L["Rt"].cuda(), b)
    wsum = tq.tq_weight_code_sums(Wq)
    Xq8, s_x, z_x, XL1b = tq.tq_quantize_act_asym_i8(X.cuda(), b, dev(L["L1t"]))
    Y = tq.tq_w4a4_lr_gemm_a8_asym(Xq8, s_x, z_x, Wq, s_w, wsum, XL1b, dev(L["L2t"]))
    torch.cuda.synchronize()
    o = oracle.layer_asym(X, L["L1t"], L["L2t"], L["Rt"], b)
    assert np.array_equal(wsum.cpu().numpy(), o["wsum"])
    q = Xq8.cpu().numpy().astype(np.int64) + 8
    assert q.min() >= 0 and q.max() <= 15
    fx = check_codes(q, o["qa"], o["t_x"], f"{name}: asymmetric codes", packed=False)
    sx, zx = s_x.cpu().numpy().astype(np.float64), z_x.cpu().numpy().astype(np.float64)
    assert np.allclose(sx, o["s_x"], rtol=2e-6, atol=0), name
    assert np.all(np.abs(zx - o["z_x"]) <= 2e-6 * (np.abs(o["z_x"]) + 15 * o["s_x"])), name
    # Y against the oracle's fp64 Y, or, where the codes hold allowed
    # midpoint flips (rows offset from zero meet exact ties v/s = k + 1/2),
    # against the definition evaluated on these codes
    if fx > 0:
        acc = q @ o["qw"].astype(np.int64).T
        want = (o["s_x"][:, None] * acc + o["z_x"][:, None] * o["wsum"][None, :]) * o["s_w"][None, :]
        if r:
            want = want + o["lr"]
    else:
        want = o["Y64"]
    fro, mx = check_y(Y.double().cpu().numpy(), want, name)
    print(f"{name}: flips {fx:.1e} fro {fro:.2e} max {mx:.2e}")


@pytest.mark.gpu
def test_asym_reduces_error_on_offset_rows(tq):
    """Rows with a mean far from zero waste half of a symmetric grid: the
    asymmetric codes reproduce the unquantized layer more closely."""
    sh = synth.CONFIGS["decode"].with_(M=256, K=1024, N=256, r=0, had_block=1)
    L = synth.make_layer(sh, seed=9)
    X = (L["X"].float() * 0.25 + 3.0).to(torch.bfloat16)  # every row offset, no rotation
    exact = X.double().numpy() @ L["Rt"].double().numpy().T
    Wq, s_w = tq.tq_pack_weight(L["Rt"].cuda(), 1)
    Xs8, s_s, _ = tq.tq_quantize_act_i8(X.cuda(), 1)
    Ys = tq.tq_w4a4_lr_gemm_a8(Xs8, s_s, Wq, s_w)
    Xa8, s_a, z_a, _ = tq.tq_quantize_act_asym_i8(X.cuda(), 1)
    Ya = tq.tq_w4a4_lr_gemm_a8_asym(Xa8, s_a, z_a, Wq, s_w, tq.tq_weight_code_sums(Wq))
    torch.cuda.synchronize()
    es = np.linalg.norm(Ys.double().cpu().numpy() - exact)
    ea = np.linalg.norm(Ya.double().cpu().numpy() - exact)
    assert ea < es, (ea, es)
