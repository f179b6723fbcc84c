"""The INT4 low-rank branch (TwinQuant Figure 4): the oracle's layer_qlr
pinned on CPU by exact properties, then tq_pack_lowrank_q4 +
tq_quantize_act_qlr_i8 + tq_w4a4_lr_gemm_a8_qlr against it, stage by stage
(each stage compared on the GPU's own upstream codes)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_y


def _layer(M=12, K=256, N=64, r=16, b=64, seed=4):
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    return synth.make_layer(sh, seed=seed)


def test_qlr_main_term_is_the_plain_layer():
    L = _layer()
    o, p = oracle.layer_qlr(L["X"], L["L1t"], L["L2t"], L["Rt"], 64), \
        oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], 64)
    assert np.array_equal(o["acc"], p["acc"]) and np.array_equal(o["qx"], p["qx"])
    main = o["s_x"][:, None] * o["s_w"][None, :] * o["acc"]
    assert np.allclose(main, p["Y64"] - p["lr"], rtol=1e-12, atol=1e-14)


def test_qlr_scales_exactly():
    """Doubling X, L1 or L2 (exact in bf16) doubles the matching scales and
    leaves every code unchanged, so Y scales exactly as the algebra says."""
    L = _layer(seed=5)
    X, L1t, L2t, Rt = (L[k].double().numpy() for k in ("X", "L1t", "L2t", "Rt"))
    o = oracle.layer_qlr(X, L1t, L2t, Rt, 64)
    lr = o["Y64"] - o["s_x"][:, None] * o["s_w"][None, :] * o["acc"]
    for name, args, want in [
            ("X", (2 * X, L1t, L2t, Rt), 2 * o["Y64"]),
            ("L1", (X, 2 * L1t, L2t, Rt), o["Y64"] + lr),
            ("L2", (X, L1t, 2 * L2t, Rt), o["Y64"] + lr)]:
        o2 = oracle.layer_qlr(*args, 64)
        assert np.array_equal(o2["qxl1"], o["qxl1"]) and np.array_equal(o2["qL2"], o["qL2"]), name
        assert np.allclose(o2["Y64"], want, rtol=1e-12, atol=1e-12 * np.abs(want).max()), name


def test_qlr_rank_permutation_invariant():
    """Permuting the r columns of L1 and of L2^T the same way permutes the
    branch's terms only: Y is unchanged."""
    L = _layer(seed=6)
    X, L1t, L2t, Rt = (L[k].double().numpy() for k in ("X", "L1t", "L2t", "Rt"))
    perm = np.random.default_rng(0).permutation(L1t.shape[0])
    a = oracle.layer_qlr(X, L1t, L2t, Rt, 64)
    c = oracle.layer_qlr(X, L1t[perm], L2t[:, perm], Rt, 64)
    assert np.allclose(a["Y64"], c["Y64"], rtol=1e-12, atol=1e-12 * np.abs(a["Y64"]).max())


def test_qlr_branch_tracks_the_bf16_branch():
    """A sanity bound, not an identity: three INT4 quantizations keep the
    branch within a few tens of percent of X L1 L2 on these factors."""
    L = _layer(M=64, K=512, N=128, r=32, b=128, seed=8)
    o = oracle.layer_qlr(L["X"], L["L1t"], L["L2t"], L["Rt"], 128)
    lr_q = o["Y64"] - o["s_x"][:, None] * o["s_w"][None, :] * o["acc"]
    exact = L["X"].double().numpy() @ L["L1t"].double().numpy().T @ L["L2t"].double().numpy().T
    assert np.linalg.norm(lr_q - exact) <= 0.3 * np.linalg.norm(exact)


@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


CASES = [
    # name, M, K, N, r, b
    ("tiles", 300, 1024, 256, 64, 128),
    ("decode_like", 16, 1024, 384, 32, 128),
    ("one_token", 1, 512, 128, 16, 64),
    ("wide_rank", 150, 512, 256, 128, 32),
    ("rank256_ragged_k", 200, 640, 256, 256, 128),   # widest fused requantization, 5 k-blocks
    ("rank272_chunked", 130, 384, 288, 272, 128),     # INT32 sums in two column launches
    ("rank512_chunked", 64, 1024, 512, 512, 64),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,K,N,r,b", CASES, ids=[c[0] for c in CASES])
def test_qlr_path_matches_oracle(tq, name, M, K, N, r, b):
    L = _layer(M=M, K=K, N=N, r=r, b=b, seed=9)
    X, L1t, L2t = L["X"].cuda(), L["L1t"].cuda(), L["L2t"].cuda()
    Wq, s_w = tq.tq_pack_weight(L["Rt"].cuda(), b)
    qL1, s_L1, qL2, s_L2 = tq.tq_pack_lowrank_q4(L1t, L2t, b)
    Xq8, s_x, XL1q, s_xl1 = tq.tq_quantize_act_qlr_i8(X, b, qL1, s_L1)
    Y = tq.tq_w4a4_lr_gemm_a8_qlr(Xq8, s_x, Wq, s_w, XL1q, s_xl1, qL2, s_L2)
    torch.cuda.synchronize()
    o = oracle.layer_qlr(L["X"], L["L1t"], L["L2t"], L["Rt"], b)
    # offline factors: codes under the midpoint rule, scales to fp32 precision
    gl1 = qL1.cpu().numpy().astype(np.int64)
    l1o = oracle.pack_weight(L["L1t"], b)
    check_codes(gl1, l1o["qw"], l1o["t_w"], f"{name}: L1 codes", packed=False)
    assert np.allclose(s_L1.cpu().numpy(), o["s_L1"], rtol=2e-6, atol=0)
    gl2 = qL2.float().cpu().numpy().astype(np.int64)
    check_codes(gl2, o["qL2"], o["t_L2"], f"{name}: L2 codes", packed=False)
    assert np.allclose(s_L2.cpu().numpy(), o["s_L2"], rtol=2e-6, atol=0)
    # activation codes
    qx = Xq8.cpu().numpy().astype(np.int64)
    check_codes(qx, o["qx"], o["t_x"], f"{name}: activation codes", packed=False)
    # X L1 requantized: the definition on the GPU's codes and scales
    sx = s_x.cpu().numpy().astype(np.float64)
    xl1 = sx[:, None] * s_L1.cpu().numpy().astype(np.float64)[None, :] * (qx @ gl1.astype(np.int64).T)
    rq, rs, rt = oracle.quantize_sym(xl1)
    gq = XL1q.float().cpu().numpy().astype(np.int64)
    check_codes(gq, rq, rt, f"{name}: requantized X L1 codes", packed=False)
    assert np.allclose(s_xl1.cpu().numpy(), rs, rtol=2e-6, atol=0)
    # Y: the definition on the GPU's codes and scales
    want = (sx[:, None] * o["s_w"][None, :] * (qx @ o["qw"].astype(np.int64).T)
            + s_xl1.cpu().numpy().astype(np.float64)[:, None]
            * s_L2.cpu().numpy().astype(np.float64)[None, :] * (gq @ gl2.T))
    check_y(Y.double().cpu().numpy(), want, name)


@pytest.mark.gpu
def test_qlr_full_size_sampled(tq):
    """The Llama-3-8B gate/up prefill shape (2048 x 4096 -> 14336, r = 64) in
    the benchmark's launch configuration; sampled tokens and channels against
    the definition (each sampled token row carries its full K)."""
    sh = synth.CONFIGS["prefill_gateup"]
    M, K, N, r, b = sh.M, sh.K, sh.N, sh.r, sh.had_block
    L = synth.make_layer(sh, seed=11, device="cuda")
    X, L1t, L2t = L["X"].cuda(), L["L1t"].cuda(), L["L2t"].cuda()
    Wq, s_w = tq.tq_pack_weight(L["Rt"].cuda(), b)
    qL1, s_L1, qL2, s_L2 = tq.tq_pack_lowrank_q4(L1t, L2t, b)
    Xq8, s_x, XL1q, s_xl1 = tq.tq_quantize_act_qlr_i8(X, b, qL1, s_L1)
    Y = tq.tq_w4a4_lr_gemm_a8_qlr(Xq8, s_x, Wq, s_w, XL1q, s_xl1, qL2, s_L2)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 1, M // 2, M - 1], rng.choice(M, 12, replace=False)]))
    cols = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 126, replace=False)]))
    rt, ct = torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()
    a = oracle.quantize_act(L["X"][torch.from_numpy(rows)], b, None)
    qx = Xq8[rt].cpu().numpy().astype(np.int64)
    check_codes(qx, a["qx"], a["t_x"], "activation codes", packed=False)
    sx = s_x[rt].cpu().numpy().astype(np.float64)
    l1o = oracle.pack_weight(L["L1t"], b)
    gl1 = qL1.cpu().numpy().astype(np.int64)
    check_codes(gl1, l1o["qw"], l1o["t_w"], "L1 codes", packed=False)
    xl1 = sx[:, None] * s_L1.cpu().numpy().astype(np.float64)[None, :] * (qx @ gl1.T)
    rq, rs, rtie = oracle.quantize_sym(xl1)
    gq = XL1q[rt].float().cpu().numpy().astype(np.int64)
    check_codes(gq, rq, rtie, "requantized X L1 codes", packed=False)
    assert np.allclose(s_xl1[rt].cpu().numpy(), rs, rtol=2e-6, atol=0)
    w = oracle.pack_weight(L["Rt"][torch.from_numpy(cols)], b)
    gl2 = qL2[ct].float().cpu().numpy().astype(np.int64)
    want = (sx[:, None] * w["s_w"][None, :] * (qx @ w["qw"].astype(np.int64).T)
            + s_xl1[rt].cpu().numpy().astype(np.float64)[:, None]
            * s_L2[ct].cpu().numpy().astype(np.float64)[None, :] * (gq @ gl2.T))
    check_y(Y[rt][:, ct].double().cpu().numpy(), want, "prefill_gateup qlr")
