"""Gate / up pair with the SwiGLU epilogue (shared input): the oracle's
silu(g) * u pinned by closed forms on CPU, then tq_pack_gate_up +
tq_w4a4_lr_gate_up against the oracle's two layers and against the same pair
run as one ordinary layer of 2N channels."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_y, y_reference


def test_swiglu_closed_forms():
    ln3 = math.log(3.0)
    # sigmoid(ln 3) = 3/4 and sigmoid(-ln 3) = 1/4 exactly
    got = oracle.swiglu(np.array([0.0, ln3, -ln3, 50.0]), np.array([5.0, 1.0, 2.0, 1.0]))
    want = np.array([0.0, 0.75 * ln3, -0.5 * ln3, 50.0])
    assert np.allclose(got, want, rtol=1e-15, atol=1e-15)
    # silu(x) - silu(-x) = x (sigmoid(x) + sigmoid(-x) = 1)
    x = np.random.default_rng(0).normal(size=1000) * 4
    one = np.ones_like(x)
    assert np.allclose(oracle.swiglu(x, one) - oracle.swiglu(-x, one), x, rtol=0, atol=1e-13)
    # linear in u
    assert np.allclose(oracle.swiglu(x, 3 * one), 3 * oracle.swiglu(x, one), rtol=1e-15, atol=0)


@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


def _pair(sh, seed):
    g = synth.make_layer(sh, seed=seed)
    u = synth.make_layer(sh, seed=seed + 100)
    u["X"] = g["X"]  # the shared input
    return g, u


CASES = [
    # name, M, K, N, r, b
    ("prefill_like", 300, 1024, 256, 32, 128),
    ("decode_like", 16, 1024, 384, 16, 128),
    ("one_token", 1, 512, 128, 16, 64),
    ("rank0", 200, 512, 136, 0, 128),
    ("wide_rank", 150, 512, 256, 128, 32),
    ("no_rotation", 140, 512, 136, 32, 1),
    ("stream_k", 600, 2048, 1024, 32, 128),   # 64 tiles x 8 stages over the SMs
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,K,N,r,b", CASES, ids=[c[0] for c in CASES])
def test_gate_up_matches_oracle(tq, name, M, K, N, r, b):
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    g, u = _pair(sh, seed=11)
    dev = lambda t: t.cuda() if t is not None else None  # noqa: E731
    Wq_g, s_w_g = tq.tq_pack_weight(g["Rt"].cuda(), b)
    Wq_u, s_w_u = tq.tq_pack_weight(u["Rt"].cuda(), b)
    L1g, L2g = (dev(g["L1t"]), dev(g["L2t"])) if r else (None, None)
    L1u, L2u = (dev(u["L1t"]), dev(u["L2t"])) if r else (None, None)
    Wq2, s_w2, L1t2, L2t2 = tq.tq_pack_gate_up(Wq_g, s_w_g, L1g, L2g, Wq_u, s_w_u, L1u, L2u)
    X = g["X"].cuda()
    Y = tq.tq_w4a4_lr_gate_up(X, L1t2, Wq2, s_w2, L2t2, b)
    # the same pair as an ordinary layer of 2N interleaved channels
    Ycat = tq.tq_w4a4_lr_layer(X, L1t2, Wq2, s_w2, L2t2, b)
    # the pair's codes (one activation pass; the codes do not depend on the
    # rank): midpoint flips allowed
    Xq8, _, _ = tq.tq_quantize_act_i8(X, b)
    torch.cuda.synchronize()
    og = oracle.layer(g["X"], g["L1t"], g["L2t"], g["Rt"], b)
    ou = oracle.layer(u["X"], u["L1t"], u["L2t"], u["Rt"], b)
    q8 = Xq8.cpu().numpy().astype(np.int64)
    fx = check_codes(q8, og["qx"], og["t_x"], f"{name}: activation codes", packed=False)
    # references: the oracle's fp64 outputs, or, where the codes hold allowed
    # flips (one flip moves a token's whole row of both g and u), the
    # oracle's epilogue on these codes
    yg, yu = y_reference(q8, og, fx), y_reference(q8, ou, fx)
    # the interleaved layer: gate channels on even rows, up on odd rows
    yc = Ycat.double().cpu().numpy()
    check_y(yc[:, 0::2], yg, f"{name}: pair layer, gate channels")
    check_y(yc[:, 1::2], yu, f"{name}: pair layer, up channels")
    # the fused pair: silu(g) * u of those references
    want = oracle.swiglu(yg, yu)
    y = Y.double().cpu().numpy()
    # in Frobenius norm: within the layer bound, or, where a few elements
    # dominate the norm (one token), within 1.1 x what rounding the exact
    # answer to bf16 itself costs (an element-wise half-ulp bound does not
    # hold: bf16(X L1) may sit one ulp from the oracle's where the fp32 X L1
    # is near a bf16 midpoint)
    floor = np.linalg.norm(oracle.round_bf16(want) - want) / np.linalg.norm(want)
    fro = np.linalg.norm(y - want) / np.linalg.norm(want)
    assert fro <= max(2e-3, 1.1 * floor), (name, fro, floor)
    # the epilogue uses the fp32 values: closer to the fp64 reference than
    # SwiGLU applied to the two bf16-rounded outputs
    from_bf16 = oracle.swiglu(yc[:, 0::2], yc[:, 1::2])  # (the pair layer's own codes)
    e_fused = np.linalg.norm(y - want)
    e_split = np.linalg.norm(from_bf16 - want)
    assert e_fused <= 1.05 * e_split + 1e-12, (e_fused, e_split)


@pytest.mark.gpu
def test_gate_up_argument_errors(tq):
    X = torch.zeros(16, 256, dtype=torch.bfloat16, device="cuda")
    Wq2 = torch.zeros(256, 128, dtype=torch.uint8, device="cuda")
    s_w2 = torch.zeros(256, dtype=torch.float32, device="cuda")
    L1t2 = torch.zeros(48, 256, dtype=torch.bfloat16, device="cuda")  # r2 = 48: not a multiple of 32
    L2t2 = torch.zeros(256, 48, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_w4a4_lr_gate_up(X, L1t2, Wq2, s_w2, L2t2, 128)
    assert e.value.status == 2
    with pytest.raises(tq.TQError) as e:
        tq.tq_w4a4_lr_gate_up(X, None, Wq2, s_w2, None, 256)  # Hadamard block above 128
    assert e.value.status == 2
