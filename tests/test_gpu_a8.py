"""Codes one per byte: tq_quantize_act_i8 + tq_w4a4_lr_gemm_a8 (and the layer
entry point that uses them for M > 128) against the fp64 oracle and against
the packed-code path."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_scales, check_y, y_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


SHAPES = [
    # name, M, K, N, r, b
    ("one_token", 1, 256, 136, 16, 128),
    ("ragged_tiles", 193, 384, 264, 48, 128),
    ("two_token_tiles", 384, 1024, 520, 64, 128),
    ("rank0", 250, 512, 128, 0, 128),
    ("rank128", 300, 2048, 256, 128, 128),
    ("one_kblock", 200, 128, 64, 16, 64),
    ("block2", 129, 256, 16, 16, 2),
    ("tiny_n", 150, 256, 8, 0, 128),
    ("no_rotation", 700, 640, 392, 32, 1),
    # ranks above 128: codes, then X L1 in launches of at most 256 columns
    ("rank144", 130, 512, 256, 144, 128),
    ("rank400", 257, 768, 512, 400, 64),
    ("rank512", 150, 1024, 640, 512, 128),
]


@pytest.mark.parametrize("name,M,K,N,r,b", SHAPES, ids=[s[0] for s in SHAPES])
def test_a8_path_matches_oracle(tq, name, M, K, N, r, b):
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, seed=5)
    X, Rt = L["X"].cuda(), L["Rt"].cuda()
    L1t = L["L1t"].cuda() if r else None
    L2t = L["L2t"].cuda() if r else None
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    Xq8, s_x, XL1b = tq.tq_quantize_act_i8(X, b, L1t)
    Y = tq.tq_w4a4_lr_gemm_a8(Xq8, s_x, Wq, s_w, XL1b, L2t)
    torch.cuda.synchronize()
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b)
    q8 = Xq8.cpu().numpy().astype(np.int64)
    assert np.abs(q8).max() <= 7
    fx = check_codes(q8, o["qx"], o["t_x"], "activation codes (int8)", packed=False)
    check_scales(s_x.cpu().numpy(), o["s_x"], "s_x")
    if r:
        # bf16 of the fp32 X L1: within one bf16 rounding of the oracle's bf16(XL1)
        xb = XL1b.float().cpu().numpy().astype(np.float64)
        ref = o["XL1"]
        assert np.all(np.abs(xb - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-5 * np.abs(ref).max())
    # Y against the oracle's fp64 Y, or, where the codes hold allowed
    # midpoint flips, against the definition evaluated on these codes
    fro, mx = check_y(Y.double().cpu().numpy(), y_reference(q8, o, fx), name)
    print(f"FLIPS a8 {name}: x={fx:.3e} fro={fro:.3e} max={mx:.3e}")


@pytest.mark.parametrize("M,K,N,b", [(256, 1024, 256, 128), (1000, 2048, 136, 2), (70, 512, 64, 128)])
def test_int8_codes_equal_packed_codes_and_integer_path_exact(tq, M, K, N, b):
    # tensor-core activation path on both sides (M >= 64): identical codes and
    # scales; with r = 0 the epilogue is the same expression on the same exact
    # integer sums, so Y must agree bit for bit with the packed-code GEMM
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=0, had_block=b)
    L = synth.make_layer(sh, seed=9)
    X, Rt = L["X"].cuda(), L["Rt"].cuda()
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    Xq, s_x, _ = tq.tq_quantize_act(X, b)
    Xq8, s_x8, _ = tq.tq_quantize_act_i8(X, b)
    torch.cuda.synchronize()
    assert np.array_equal(oracle.unpack_int4(Xq.cpu().numpy()).astype(np.int16),
                          Xq8.cpu().numpy().astype(np.int16))
    assert torch.equal(s_x, s_x8)
    Y = tq.tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w)
    Y8 = tq.tq_w4a4_lr_gemm_a8(Xq8, s_x8, Wq, s_w)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y8)


def test_layer_entry_prefill(tq):
    sh = synth.CONFIGS["decode"].with_(M=600, K=1536, N=384, r=64, had_block=128)
    L = synth.make_layer(sh, seed=11)
    X, Rt, L1t, L2t = (L[k].cuda() for k in ("X", "Rt", "L1t", "L2t"))
    Wq, s_w = tq.tq_pack_weight(Rt, 128)
    Y = tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128)
    Y2 = tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128)
    Xq8, s_x, XL1b = tq.tq_quantize_act_i8(X, 128, L1t)
    Y8 = tq.tq_w4a4_lr_gemm_a8(Xq8, s_x, Wq, s_w, XL1b, L2t)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], 128)
    check_y(Y.double().cpu().numpy(), o["Y64"], "layer entry (M > 128)")
    check_y(Y8.double().cpu().numpy(), o["Y64"], "codes one per byte")


def test_a8_argument_errors(tq):
    X = torch.zeros(256, 512, dtype=torch.bfloat16, device="cuda")
    L1t = torch.zeros(528, 512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act_i8(X, 128, L1t)  # r = 528 > 512
    assert e.value.status == 2
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act_i8(X, 256)  # had_block 256 > 128
    assert e.value.status == 2
