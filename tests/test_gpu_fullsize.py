"""Full-size layers through the C ABI, checked on sampled outputs.

The CUDA path runs the whole layer at the workload sizes (Llama-3-8B MLP
prefill, Llama-3-70B-sized MLP, the 4096^3 rank/M sweep) in the launch
configuration the benchmark times; the oracle recomputes a sample of tokens
and output channels one by one (each sampled row needs its full-K rotation and
absmax, so the sample is exact, not an approximation of the full run).
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


def _run_and_check(sh, n_rows=10, n_cols=160, seed=0):
    import rank_int4_gemm_b200 as tq
    L = synth.make_layer(sh, seed=seed, device="cuda")
    b, r = sh.had_block, sh.r
    X = L["X"].cuda()
    Rt = L["Rt"].cuda()
    L1t = L["L1t"].cuda() if r else None
    L2t = L["L2t"].cuda() if r else None
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    del Rt
    Xq, s_x, XL1 = tq.tq_quantize_act(X, b, L1t)
    Y = tq.tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed + 123)
    rows = _sample(sh.M, n_rows, rng)
    cols = _sample(sh.N, n_cols, rng)
    rows_t = torch.from_numpy(rows)
    cols_t = torch.from_numpy(cols)
    Xs = L["X"][rows_t]
    a = oracle.quantize_act(Xs, b, L["L1t"] if r else None)
    w = oracle.pack_weight(L["Rt"][cols_t], b)
    acc = oracle.int_gemm(a["qx"], w["qw"])
    lr = None
    if r:
        _, lr = oracle.lowrank(Xs, L["L1t"], L["L2t"][cols_t])
    y64 = oracle.epilogue(a["s_x"], w["s_w"], acc, lr)
    fx = check_codes(Xq[rows_t.cuda()].cpu().numpy(), a["qx"], a["t_x"], "activation codes")
    fw = check_codes(Wq[cols_t.cuda()].cpu().numpy(), w["qw"], w["t_w"], "weight codes")
    check_scales(s_x[rows_t.cuda()].cpu().numpy(), a["s_x"], "s_x")
    check_scales(s_w[cols_t.cuda()].cpu().numpy(), w["s_w"], "s_w")
    if r:
        check_xl1(XL1[rows_t.cuda()].cpu().numpy(), Xs.double().numpy(),
                  L["L1t"].double().numpy(), a["XL1"])
    ys = Y[rows_t.cuda()][:, cols_t.cuda()].double().cpu().numpy()
    fro, mx = check_y(ys, y64)
    return fx, fw, fro, mx


@pytest.mark.parametrize("name", ["prefill_gateup", "prefill_down"])
def test_prefill_llama3_8b_mlp(cuda_ok, name):
    fx, fw, fro, mx = _run_and_check(synth.CONFIGS[name])
    print(f"{name}: flips x={fx:.1e} w={fw:.1e} fro={fro:.2e} max={mx:.2e}")


@pytest.mark.parametrize("name", ["large_gateup", "large_down"])
def test_large_llama3_70b_mlp(cuda_ok, name):
    fx, fw, fro, mx = _run_and_check(synth.CONFIGS[name], n_rows=6, n_cols=96)
    print(f"{name}: flips x={fx:.1e} w={fw:.1e} fro={fro:.2e} max={mx:.2e}")


@pytest.mark.parametrize("r", [0, 512])
def test_sweep_rank_extremes(cuda_ok, r):
    _run_and_check(synth.CONFIGS["sweep"].with_(r=r))


@pytest.mark.parametrize("M", [1, 4, 64, 256, 8192])
def test_sweep_token_counts(cuda_ok, M):
    _run_and_check(synth.CONFIGS["sweep"].with_(M=M), n_rows=min(M, 8))
