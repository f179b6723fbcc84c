"""tq_w4a4_lr_layer (bf16 X -> Y in one call; one fused kernel at decode
sizes) against the fp64 oracle and against the two-call path."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_y

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


CASES = [
    # name, M, K, N, r, b      (fused: M<=16, r in {0,16,32,64}, K%256==0, K<=4096, b<=256)
    ("decode_m1", 1, 4096, 4096, 32, 128),
    ("decode_m3", 3, 4096, 4096, 32, 128),
    ("decode_m16", 16, 4096, 4096, 32, 128),
    ("one_split", 16, 512, 256, 16, 128),
    ("ragged_splits", 5, 1536, 136, 16, 128),
    ("rank0", 7, 2048, 264, 0, 128),
    ("rank0_decode_m16", 16, 4096, 4096, 0, 128),
    ("rank0_block32", 13, 1024, 256, 0, 32),
    ("rank64_block256", 16, 4096, 512, 64, 256),
    ("no_rotation", 2, 1024, 128, 32, 1),
    ("block2", 9, 1024, 384, 48, 2),
    ("block16", 4, 1024, 256, 16, 16),
    ("block64", 11, 2048, 384, 32, 64),
    # two-kernel path inside the same entry point
    ("fallback_m17", 17, 1024, 256, 32, 128),
    ("fallback_rank128", 8, 1024, 256, 128, 128),
    ("fallback_k384", 4, 384, 136, 16, 128),
    ("fallback_k8192", 16, 8192, 512, 64, 256),
]


@pytest.mark.parametrize("name,M,K,N,r,b", CASES, ids=[c[0] for c in CASES])
def test_layer_entry_matches_oracle_and_two_call_path(tq, name, M, K, N, r, b):
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, device="cuda" if K * N >= 1 << 22 else "cpu")
    X, Rt = L["X"].cuda(), L["Rt"].cuda()
    L1t = L["L1t"].cuda() if r else None
    L2t = L["L2t"].cuda() if r else None
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    y_one = tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, b)
    y_two = tq.layer_forward(X, L1t, L2t, Wq, s_w, b)
    torch.cuda.synchronize()
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b)
    check_y(y_one.double().cpu().numpy(), o["Y64"], f"{name}: layer entry vs oracle")
    if r == 0:
        # no low-rank branch: the same codes, scales and exact integer sums
        # meet the same fp32 epilogue on both paths, so Y is equal bit for bit
        assert torch.equal(y_one, y_two), f"{name}: {(y_one.float() - y_two.float()).abs().max()}"
    else:
        # same codes and scales on both paths; only the X L1 summation order
        # differs, which moves bf16(X L1) by at most one bf16 ulp
        a, c = y_one.double().cpu().numpy(), y_two.double().cpu().numpy()
        tol = 2.0 ** -7 * np.abs(c) + 1e-3 * np.abs(c).max()
        assert np.all(np.abs(a - c) <= tol), f"{name}: {np.abs(a - c).max()}"


def test_layer_entry_tiny_row(tq):
    sh = synth.CONFIGS["decode"].with_(M=4, K=1024, N=256, r=32)
    L = synth.make_layer(sh)
    L["X"][1] = (L["X"][1].float() * 2.0 ** -110).to(torch.bfloat16)  # absmax ~1e-31
    X, Rt, L1t, L2t = (L[k].cuda() for k in ("X", "Rt", "L1t", "L2t"))
    Wq, s_w = tq.tq_pack_weight(Rt, 128)
    y = tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128)
    torch.cuda.synchronize()
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], 128)
    check_y(y.double().cpu().numpy(), o["Y64"], "tiny row")
    # the tiny row on its own scale
    y1, o1 = y[1].double().cpu().numpy(), o["Y64"][1]
    assert np.linalg.norm(y1 - o1) <= 2e-3 * np.linalg.norm(o1)


def test_layer_entry_deterministic(tq):
    sh = synth.CONFIGS["decode"].with_(M=16, K=4096, N=1024, r=32)
    L = synth.make_layer(sh, device="cuda")
    X, Rt, L1t, L2t = (L[k].cuda() for k in ("X", "Rt", "L1t", "L2t"))
    Wq, s_w = tq.tq_pack_weight(Rt, 128)
    a = tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128)
    b = tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
