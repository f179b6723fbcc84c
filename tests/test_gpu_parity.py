"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Sizes are small enough for the oracle to finish in seconds yet span several
tiles and ragged tails; the decode layer (K = N = 4096, M in {1, 16, 128}) is
checked in full.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_scales, check_xl1, check_y

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


def _dev(t):
    return t.contiguous().cuda()


def _run_layer(tq, L, b):
    X, L1t, L2t, Rt = (_dev(L[k]) for k in ("X", "L1t", "L2t", "Rt"))
    r = L1t.shape[0]
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    Xq, s_x, XL1 = tq.tq_quantize_act(X, b, L1t if r else None)
    Y = tq.tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t if r else None)
    torch.cuda.synchronize()
    return {k: (v.cpu() if v is not None else None)
            for k, v in dict(Wq=Wq, s_w=s_w, Xq=Xq, s_x=s_x, XL1=XL1, Y=Y).items()}


def _check_layer(g, L, b):
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b)
    fw = check_codes(g["Wq"].numpy(), o["qw"], o["t_w"], "weight codes")
    fx = check_codes(g["Xq"].numpy(), o["qx"], o["t_x"], "activation codes")
    check_scales(g["s_w"].numpy(), o["s_w"], "s_w")
    check_scales(g["s_x"].numpy(), o["s_x"], "s_x")
    if L["L1t"].shape[0]:
        check_xl1(g["XL1"].numpy(), L["X"].double().numpy(), L["L1t"].double().numpy(), o["XL1"])
    fro, mx = check_y(g["Y"].double().numpy(), o["Y64"])
    return fw, fx, fro, mx


SHAPES = [
    # name, M, K, N, r, b
    ("tiny", 16, 256, 256, 16, 256),
    ("ragged_small", 17, 384, 136, 16, 128),
    ("multi_tile", 300, 512, 520, 32, 128),
    ("rank0", 40, 256, 264, 0, 64),
    ("min_sizes", 1, 128, 8, 0, 128),
    ("min_rank", 3, 128, 16, 16, 128),
    ("block2", 5, 256, 64, 16, 2),
    ("no_rotation", 130, 256, 128, 32, 1),
    ("big_rank", 9, 1024, 512, 512, 128),
]


# tq_quantize_act on tensor cores (M >= 64, b <= 128): 128-token tiles,
# ragged last tile, one and several CTAs along K, every block size; ranks
# above 128 (codes, then X L1 in launches of at most 256 columns)
TC_SHAPES = [
    ("tc_min_m", 64, 256, 128, 16, 128),
    ("tc_ragged", 129, 1024, 136, 32, 128),
    ("tc_one_block", 200, 128, 64, 16, 128),
    ("tc_rank0", 300, 512, 264, 0, 128),
    ("tc_rank128", 140, 2048, 256, 128, 128),
    ("tc_block2", 96, 512, 128, 48, 2),
    ("tc_block64", 70, 768, 128, 64, 64),
    ("tc_no_rotation", 65, 384, 64, 16, 1),
    ("tc_many_tiles", 1100, 1536, 256, 64, 128),
    ("tc_rank256", 130, 1024, 384, 256, 128),
    ("tc_rank304", 200, 512, 384, 304, 32),
]


@pytest.mark.parametrize("name,M,K,N,r,b", TC_SHAPES, ids=[s[0] for s in TC_SHAPES])
def test_activation_tensor_core_path(tq, name, M, K, N, r, b):
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, seed=3)
    g = _run_layer(tq, L, b)
    fw, fx, fro, mx = _check_layer(g, L, b)
    print(f"{name}: flips x={fx:.1e} w={fw:.1e} fro={fro:.2e} max={mx:.2e}")


@pytest.mark.parametrize("name,M,K,N,r,b", SHAPES, ids=[s[0] for s in SHAPES])
def test_layer_small(tq, name, M, K, N, r, b):
    base = synth.CONFIGS["tiny"] if name == "tiny" else synth.CONFIGS["decode"]
    sh = base.with_(M=M, K=K, N=N, r=r, had_block=b,
                    outlier_channels=None if name != "tiny" else 2)
    L = synth.make_layer(sh)
    g = _run_layer(tq, L, b)
    _check_layer(g, L, b)


@pytest.mark.parametrize("M", [1, 16, 128])
def test_decode_layer_full(tq, M):
    sh = synth.CONFIGS["decode"].with_(M=M)
    L = synth.make_layer(sh, device="cuda")
    g = _run_layer(tq, L, sh.had_block)
    fw, fx, fro, mx = _check_layer(g, L, sh.had_block)
    print(f"decode M={M}: flips w={fw:.2e} x={fx:.2e} fro={fro:.2e} max={mx:.2e}")


ACC_SHAPES = [(1, 128, 128), (16, 256, 256), (17, 384, 136), (128, 512, 264),
              (129, 256, 512), (300, 1024, 520), (64, 4096, 4096), (256, 32768, 64)]


@pytest.mark.parametrize("M,K,N", ACC_SHAPES)
def test_int32_accumulators_bit_exact(tq, M, K, N):
    # Codes of the oracle's choice (uniform in [-7, 7], plus rows at the
    # extremes) go through the GEMM kernel's integer path unchanged.
    rng = np.random.default_rng(M * 7 + K + N)
    qa = rng.integers(-7, 8, size=(M, K)).astype(np.int8)
    qb = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    qa[0, :] = 7
    qb[-1, :] = -7
    if M > 1:
        qa[-1, :] = -7
    want = oracle.int_gemm(qa, qb)
    Xq = torch.from_numpy(oracle.pack_int4(qa)).cuda()
    Wq = torch.from_numpy(oracle.pack_int4(qb)).cuda()
    acc = tq.tq_debug_w4a4_gemm_acc(Xq, Wq)
    torch.cuda.synchronize()
    got = acc.cpu().numpy().astype(np.int64)
    assert np.array_equal(got, want)


def test_gemm_on_oracle_codes_is_bf16_close(tq):
    # Same codes and scales on both sides: the only differences left are the
    # fp32 epilogue and the final bf16 rounding, so every element agrees with
    # the fp64 value to within one bf16 ulp (plus fp32 noise of the low-rank
    # sum, bounded by 1e-5 of its absolute terms).
    sh = synth.CONFIGS["decode"].with_(M=200, K=512, N=392, r=48)
    L = synth.make_layer(sh)
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], sh.had_block)
    Xq = torch.from_numpy(o["Xq"]).cuda()
    Wq = torch.from_numpy(o["Wq"]).cuda()
    s_x = torch.from_numpy(o["s_x"].astype(np.float32)).cuda()
    s_w = torch.from_numpy(o["s_w"].astype(np.float32)).cuda()
    XL1 = torch.from_numpy(o["XL1"].astype(np.float32)).cuda()
    L2t = L["L2t"].cuda()
    Y = tq.tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t)
    torch.cuda.synchronize()
    y = Y.cpu().double().numpy()
    # oracle epilogue on the fp32-rounded scales and XL1 the kernel was given
    lr = oracle.round_bf16(o["XL1"].astype(np.float32).astype(np.float64)) @ L["L2t"].double().numpy().T
    y64 = oracle.epilogue(o["s_x"].astype(np.float32), o["s_w"].astype(np.float32), o["acc"], lr)
    lr_abs = np.abs(oracle.round_bf16(o["XL1"].astype(np.float32).astype(np.float64))) @ \
        np.abs(L["L2t"].double().numpy()).T
    tol = 2.0 ** -8 * np.abs(y64) + 1e-5 * lr_abs + 4e-7 * np.abs(y64) + 1e-30
    assert np.all(np.abs(y - y64) <= tol)


def test_zero_rows_and_channels(tq):
    sh = synth.CONFIGS["decode"].with_(M=20, K=256, N=128, r=16)
    L = synth.make_layer(sh)
    L["X"][3] = 0
    L["Rt"][5] = 0
    g = _run_layer(tq, L, 128)
    assert g["s_x"][3] == 0 and not g["Xq"][3].any()
    assert g["s_w"][5] == 0 and not g["Wq"][5].any()
    _check_layer(g, L, 128)


def test_tiny_rows(tq):
    # rows whose absmax is far below 1 (down to ~1e-36): 7 / absmax would
    # overflow fp32 without the kernel's exact power-of-two prescale
    sh = synth.CONFIGS["decode"].with_(M=12, K=512, N=128, r=16)
    L = synth.make_layer(sh)
    L["X"][2] = (L["X"][2].float() * 2.0 ** -120).to(torch.bfloat16)
    L["X"][7] = (L["X"][7].float() * 2.0 ** -60).to(torch.bfloat16)
    assert L["X"][2].abs().max() > 0
    g = _run_layer(tq, L, 128)
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], 128)
    check_codes(g["Xq"].numpy(), o["qx"], o["t_x"], "activation codes")
    check_scales(g["s_x"].numpy(), o["s_x"], "s_x")
    assert g["Xq"][2].any() and g["Xq"][7].any()


def test_deterministic(tq):
    sh = synth.CONFIGS["decode"].with_(M=16, K=1024, N=512, r=32)
    L = synth.make_layer(sh)
    a = _run_layer(tq, L, 128)
    b = _run_layer(tq, L, 128)
    for k in ("Wq", "s_w", "Xq", "s_x", "XL1", "Y"):
        assert torch.equal(a[k], b[k]), k


def test_argument_errors_before_launch(tq):
    X = torch.zeros(4, 100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.TQError) as e:
        tq.tq_quantize_act(X, 128)
    assert e.value.status == 2  # TQ_ERR_UNSUPPORTED_SHAPE
