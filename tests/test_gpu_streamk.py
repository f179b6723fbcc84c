"""The codes-one-per-byte GEMM under its stream-K schedule: with the scratch
in the workspace the persistent CTAs split tiles x k-blocks evenly, and a
split tile is finished by the CTA holding its first k-blocks from the other
CTAs' INT32 partial sums.  Integer addition is exact, so Y must equal the
tile-by-tile schedule's Y (a 256-byte workspace) bit for bit, on shapes
where tiles are split between two CTAs, among ten, with an odd number of
k-blocks and with the low-rank stages only in the finishing CTA; and Y
must meet the oracle's tolerance.  After each call the ready flags are zero
again, so repeated calls give the same Y."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_y, y_reference

pytestmark = pytest.mark.gpu

FLAG_BYTES = 160 * 8 * 4   # the scratch's flag words come first


@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


SHAPES = [
    # name, M, K, N, r, b
    ("ten_ctas_per_tile", 384, 8192, 1024, 0, 128),       # 16 tiles, 32 stages each
    ("odd_kblocks", 200, 4224, 2056, 32, 128),            # 33 k-blocks, ragged N tile
    ("two_ctas_per_tile", 1000, 2048, 4096, 64, 128),     # 192 tiles over 148 CTAs
    ("rank128", 600, 3072, 1536, 128, 64),
    ("ragged_tokens", 1100, 1024, 1536, 16, 128),
]


def _inputs(tq, M, K, N, r, b, seed=11):
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, seed=seed)
    X, Rt = L["X"].cuda(), L["Rt"].cuda()
    L1t = L["L1t"].cuda() if r else None
    L2t = L["L2t"].cuda() if r else None
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    Xq8, s_x, XL1b = tq.tq_quantize_act_i8(X, b, L1t)
    return L, Wq, s_w, Xq8, s_x, XL1b, L2t


def _ws(tq, M, N, K, r):
    return torch.zeros(tq.tq_gemm_a8_workspace_bytes(M, N, K, r), dtype=torch.uint8,
                       device="cuda")


@pytest.mark.parametrize("name,M,K,N,r,b", SHAPES, ids=[s[0] for s in SHAPES])
def test_stream_k_equals_tile_schedule_and_oracle(tq, name, M, K, N, r, b):
    L, Wq, s_w, Xq8, s_x, XL1b, L2t = _inputs(tq, M, K, N, r, b)
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    Y_dp = tq.tq_w4a4_lr_gemm_a8(Xq8, s_x, Wq, s_w, XL1b, L2t, workspace=small)
    ws = _ws(tq, M, N, K, r)
    Y_sk = tq.tq_w4a4_lr_gemm_a8(Xq8, s_x, Wq, s_w, XL1b, L2t, workspace=ws)
    torch.cuda.synchronize()
    flags = ws[256:256 + FLAG_BYTES]
    part = ws[256 + FLAG_BYTES:]
    assert int(part.count_nonzero()) > 0, "no partial tile was written: stream-K did not run"
    assert int(flags.count_nonzero()) == 0, "ready flags left set"
    assert torch.equal(Y_sk, Y_dp)
    Y_sk2 = tq.tq_w4a4_lr_gemm_a8(Xq8, s_x, Wq, s_w, XL1b, L2t, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(Y_sk2, Y_sk)
    assert tq.tq_query_device_status(ws) == 0
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b)
    q8 = Xq8.cpu().numpy().astype(np.int64)
    fx = check_codes(q8, o["qx"], o["t_x"], "activation codes (int8)", packed=False)
    fro, mx = check_y(Y_sk.double().cpu().numpy(), y_reference(q8, o, fx), name)
    print(f"FLIPS streamk {name}: x={fx:.3e} fro={fro:.3e} max={mx:.3e}")


def test_stream_k_integer_sums_bit_exact(tq):
    # r = 0, s_x = s_w = 1: Y = bf16(sum q q), and bf16 holds every integer
    # up to 256 exactly.  Each token has four nonzero codes, at columns spread
    # over K (so the k-blocks of several CTAs contribute), hence |sum| <= 196
    # and Y must be the oracle's integer product exactly
    M, K, N = 384, 6144, 512
    g = torch.Generator().manual_seed(3)
    q8 = torch.zeros(M, K, dtype=torch.int8)
    cols = torch.randint(0, K, (M, 4), generator=g)
    vals = torch.randint(-7, 8, (M, 4), generator=g, dtype=torch.int8)
    for i in range(4):
        q8[torch.arange(M), cols[:, i]] = vals[:, i]
    qw = torch.randint(-7, 8, (N, K), generator=g, dtype=torch.int8)
    Wq = torch.from_numpy(oracle.pack_int4(qw.numpy()))
    ref = oracle.int_gemm(q8.numpy(), qw.numpy())
    assert np.abs(ref).max() <= 256 and np.count_nonzero(ref) > M * N // 2
    ones_m = torch.ones(M, dtype=torch.float32, device="cuda")
    ones_n = torch.ones(N, dtype=torch.float32, device="cuda")
    ws = _ws(tq, M, N, K, 0)
    Y = tq.tq_w4a4_lr_gemm_a8(q8.cuda(), ones_m, Wq.cuda(), ones_n, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[256 + FLAG_BYTES:].count_nonzero()) > 0
    assert np.array_equal(Y.float().cpu().numpy().astype(np.int64), ref)


def test_stream_k_other_epilogues_equal_tile_schedule(tq):
    # asymmetric codes and the INT4 low-rank branch add the same partial sums
    # before their own epilogues
    M, K, N, r, b = 700, 4096, 1024, 32, 128
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, seed=21)
    X, Rt = L["X"].cuda(), L["Rt"].cuda()
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    L1t, L2t = L["L1t"].cuda(), L["L2t"].cuda()
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    Xa8, s_a, z_a, XL1a = tq.tq_quantize_act_asym_i8(X, b, L1t)
    wsum = tq.tq_weight_code_sums(Wq)
    Ya_dp = tq.tq_w4a4_lr_gemm_a8_asym(Xa8, s_a, z_a, Wq, s_w, wsum, XL1a, L2t, workspace=small)
    Ya_sk = tq.tq_w4a4_lr_gemm_a8_asym(Xa8, s_a, z_a, Wq, s_w, wsum, XL1a, L2t,
                                       workspace=_ws(tq, M, N, K, r))
    qL1, s_L1, qL2, s_L2 = tq.tq_pack_lowrank_q4(L1t, L2t, b)
    Xq8, s_x, XL1q, s_xl1 = tq.tq_quantize_act_qlr_i8(X, b, qL1, s_L1)
    Yq_dp = tq.tq_w4a4_lr_gemm_a8_qlr(Xq8, s_x, Wq, s_w, XL1q, s_xl1, qL2, s_L2, workspace=small)
    Yq_sk = tq.tq_w4a4_lr_gemm_a8_qlr(Xq8, s_x, Wq, s_w, XL1q, s_xl1, qL2, s_L2,
                                      workspace=_ws(tq, M, N, K, r))
    torch.cuda.synchronize()
    assert torch.equal(Ya_sk, Ya_dp)
    assert torch.equal(Yq_sk, Yq_dp)


def test_layer_entry_takes_stream_k(tq):
    # the layer entry (M > 128) carries the scratch in its workspace; its Y
    # equals the two calls with the tile schedule (the gate/up pair's
    # stream-K case is in its own test file, against the oracle)
    M, K, N, r, b = 520, 2048, 2048, 32, 128
    L, Wq, s_w, Xq8, s_x, XL1b, L2t = _inputs(tq, M, K, N, r, b, seed=4)
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    Y_dp = tq.tq_w4a4_lr_gemm_a8(Xq8, s_x, Wq, s_w, XL1b, L2t, workspace=small)
    Y_layer = tq.tq_w4a4_lr_layer(L["X"].cuda(), L["L1t"].cuda(), Wq, s_w, L2t, b)
    torch.cuda.synchronize()
    assert tq.tq_layer_path(M, N, K, r, b) == "codes_i8"
    assert torch.equal(Y_layer, Y_dp)
