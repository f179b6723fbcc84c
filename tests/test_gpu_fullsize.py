"""Full-size layers through the C ABI, checked on sampled outputs.

Each workload shape (Llama-3-8B MLP prefill, the Llama-3-70B-sized MLP, the
4096^3 rank and token sweeps) runs at its full size on the GPU; the oracle
recomputes a sample of tokens and output channels one by one (each sampled
row needs its full-K rotation and absmax, so the sample is exact, not an
approximation of the full run).

Two call sequences are covered:

* ``i8``: tq_quantize_act_i8 + tq_w4a4_lr_gemm_a8 (codes one per byte), the
  kernels tq_w4a4_lr_layer runs for M > 128 with a Hadamard block <= 128 and
  the ones the benchmark's prefill legs time, with the same arguments;
* ``packed``: tq_quantize_act + tq_w4a4_lr_gemm (packed codes), the
  kernels tq_w4a4_lr_layer runs for the other shapes (few tokens, or a
  Hadamard block of 256).

Y is compared with the oracle's fp64 Y at the layer tolerance (relative
Frobenius 2e-3, max-abs 1e-2 max|Y|); codes under the midpoint rule.  Each
case prints its midpoint-flip fraction (``FLIPS`` lines).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_scales, check_xl1, check_y

pytestmark = pytest.mark.gpu


def _sample(n, k, rng):
    base = {i for i in (0, 1, n - 1, n - 2, n // 2) if 0 <= i < n}
    extra = rng.choice(n, size=min(n, k), replace=False)
    return np.array(sorted(base | set(int(v) for v in extra)))


def _run_and_check(sh, path, n_rows=10, n_cols=160, seed=0):
    import rank_int4_gemm_b200 as tq
    L = synth.make_layer(sh, seed=seed, device="cuda")
    b, r = sh.had_block, sh.r
    X = L["X"].cuda()
    Rt = L["Rt"].cuda()
    L1t = L["L1t"].cuda() if r else None
    L2t = L["L2t"].cuda() if r else None
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    del Rt
    if path == "i8":
        assert tq.tq_layer_path(sh.M, sh.N, sh.K, r, b) == "codes_i8"
        Xq8, s_x, XL1b = tq.tq_quantize_act_i8(X, b, L1t)
        Y = tq.tq_w4a4_lr_gemm_a8(Xq8, s_x, Wq, s_w, XL1b, L2t)
    else:
        Xq, s_x, XL1 = tq.tq_quantize_act(X, b, L1t)
        Y = tq.tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed + 123)
    rows = _sample(sh.M, n_rows, rng)
    cols = _sample(sh.N, n_cols, rng)
    rows_t = torch.from_numpy(rows)
    cols_t = torch.from_numpy(cols)
    rows_c, cols_c = rows_t.cuda(), cols_t.cuda()
    Xs = L["X"][rows_t]
    a = oracle.quantize_act(Xs, b, L["L1t"] if r else None)
    w = oracle.pack_weight(L["Rt"][cols_t], b)
    acc = oracle.int_gemm(a["qx"], w["qw"])
    lr = None
    if r:
        _, lr = oracle.lowrank(Xs, L["L1t"], L["L2t"][cols_t])
    y64 = oracle.epilogue(a["s_x"], w["s_w"], acc, lr)
    if path == "i8":
        q8 = Xq8[rows_c].cpu().numpy().astype(np.int64)
        assert np.abs(q8).max() <= 7
        fx = check_codes(q8, a["qx"], a["t_x"], "activation codes (int8)", packed=False)
        if r:
            xb = XL1b[rows_c].float().cpu().numpy().astype(np.float64)
            ref = a["XL1"]
            # bf16 of the fp32 X L1: one bf16 rounding from the oracle's value
            assert np.all(np.abs(xb - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-5 * np.abs(ref).max())
    else:
        fx = check_codes(Xq[rows_c].cpu().numpy(), a["qx"], a["t_x"], "activation codes")
        if r:
            check_xl1(XL1[rows_c].cpu().numpy(), Xs.double().numpy(),
                      L["L1t"].double().numpy(), a["XL1"])
    fw = check_codes(Wq[cols_c].cpu().numpy(), w["qw"], w["t_w"], "weight codes")
    check_scales(s_x[rows_c].cpu().numpy(), a["s_x"], "s_x")
    check_scales(s_w[cols_c].cpu().numpy(), w["s_w"], "s_w")
    ys = Y[rows_c][:, cols_c].double().cpu().numpy()
    fro, mx = check_y(ys, y64)
    print(f"FLIPS {sh.name} M={sh.M} K={sh.K} N={sh.N} r={r} path={path}: "
          f"x={fx:.3e} w={fw:.3e} fro={fro:.3e} max={mx:.3e}")
    return fx, fw, fro, mx


@pytest.mark.parametrize("name", ["prefill_gateup", "prefill_down"])
def test_prefill_llama3_8b_mlp_i8(cuda_ok, name):
    _run_and_check(synth.CONFIGS[name], "i8")


@pytest.mark.parametrize("name", ["large_gateup", "large_down"])
def test_large_llama3_70b_mlp_i8(cuda_ok, name):
    _run_and_check(synth.CONFIGS[name], "i8", n_rows=6, n_cols=96)


@pytest.mark.parametrize("M", [4096, 8192])
def test_sweep_many_tokens_i8(cuda_ok, M):
    _run_and_check(synth.CONFIGS["sweep"].with_(M=M), "i8", n_rows=8)


@pytest.mark.parametrize("r", [0, 512])
def test_sweep_rank_extremes_i8(cuda_ok, r):
    _run_and_check(synth.CONFIGS["sweep"].with_(r=r), "i8")


@pytest.mark.parametrize("name", ["prefill_gateup", "prefill_down"])
def test_prefill_llama3_8b_mlp_packed(cuda_ok, name):
    _run_and_check(synth.CONFIGS[name], "packed")


@pytest.mark.parametrize("r", [0, 512])
def test_sweep_rank_extremes_packed(cuda_ok, r):
    _run_and_check(synth.CONFIGS["sweep"].with_(r=r), "packed")


@pytest.mark.parametrize("M", [1, 4, 64])
def test_sweep_few_tokens_packed(cuda_ok, M):
    _run_and_check(synth.CONFIGS["sweep"].with_(M=M), "packed", n_rows=min(M, 8))


def test_block256_many_tokens_packed(cuda_ok):
    # a Hadamard block of 256 keeps the packed-code kernels for any M
    _run_and_check(synth.CONFIGS["sweep"].with_(M=1024, had_block=256), "packed", n_rows=8)
