"""Shared-input projections (Q, K and V of Llama-3-8B attention: K = 4096,
N_q = 4096, N_k = N_v = 1024 under grouped-query attention), packed by
tq_pack_shared_input into one layer and run through tq_w4a4_lr_layer: one
activation pass, one GEMM.  Each projection's column slice of Y is checked
against the oracle's layer for that projection alone (CoQuant Eq. (14):
layers sharing an input share one transform), and the packing itself is
checked byte for byte on the host."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity_util import check_codes, check_y, y_reference

ROOT_SHAPES = {"q": 4096, "k": 1024, "v": 1024}


def _projections(M, K, Ns, rs, b, seed):
    out = []
    for i, (N, r) in enumerate(zip(Ns, rs)):
        sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
        out.append(synth.make_layer(sh, seed=seed + 17 * i, device="cuda" if K * N >= 1 << 22 else "cpu"))
    X = out[0]["X"]
    for L in out:
        L["X"] = X  # one input
    return X, out


@pytest.fixture(scope="module")
def tq(cuda_ok):
    import rank_int4_gemm_b200 as m
    return m


CASES = [
    # name, M, K, (N_q, N_k, N_v), (r_q, r_k, r_v), b
    ("llama3_8b_decode", 16, 4096, (4096, 1024, 1024), (32, 32, 32), 128),
    ("llama3_8b_prefill", 300, 4096, (4096, 1024, 1024), (32, 32, 32), 128),
    ("one_token", 1, 4096, (4096, 1024, 1024), (32, 32, 32), 128),
    ("mixed_ranks", 140, 1024, (512, 256, 256), (64, 16, 0), 64),
    ("no_lowrank", 20, 2048, (1024, 512, 512), (0, 0, 0), 128),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,M,K,Ns,rs,b", CASES, ids=[c[0] for c in CASES])
def test_shared_input_projections_match_oracle(tq, name, M, K, Ns, rs, b):
    X, lays = _projections(M, K, Ns, rs, b, seed=40)
    packed = []
    for L, r in zip(lays, rs):
        Wq, s_w = tq.tq_pack_weight(L["Rt"].cuda(), b)
        packed.append((Wq, s_w, L["L1t"].cuda() if r else None, L["L2t"].cuda() if r else None))
    Wq_c, s_w_c, L1t_c, L2t_c, N_list = tq.tq_pack_shared_input(packed)
    Xd = X.cuda()
    Y = tq.tq_w4a4_lr_layer(Xd, L1t_c, Wq_c, s_w_c, L2t_c, b)
    torch.cuda.synchronize()
    # the packing: concatenated rows and scales, stacked L1^T, block-diagonal L2^T
    assert torch.equal(Wq_c, torch.cat([p[0] for p in packed]))
    assert torch.equal(s_w_c, torch.cat([p[1] for p in packed]))
    if sum(rs):
        assert torch.equal(L1t_c, torch.cat([p[2] for p in packed if p[2] is not None]))
        l2 = L2t_c.cpu()
        r0 = n0 = 0
        for (Wq, _, _, L2t), N, r in zip(packed, Ns, rs):
            blk = l2[n0:n0 + N]
            if r:
                assert torch.equal(blk[:, r0:r0 + r], L2t.cpu())
            rest = torch.cat([blk[:, :r0], blk[:, r0 + r:]], dim=1)
            assert not rest.float().abs().any()
            n0, r0 = n0 + N, r0 + r
    # each projection's slice against the oracle's layer for it alone
    for i, (ys, L) in enumerate(zip(tq.split_shared_output(Y, N_list), lays)):
        o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b)
        qw = oracle.unpack_int4(packed[i][0].cpu().numpy())
        fw = check_codes(qw, o["qw"], o["t_w"], f"{name}[{i}] weight codes", packed=False)
        check_y(ys.double().cpu().numpy(), y_reference(None, o, 0, qw, fw), f"{name}[{i}]")


def test_pack_shared_input_argument_checks():
    import rank_int4_gemm_b200 as tq
    lib = tq.tq.raw()
    P = ctypes.c_void_p
    FAKE = 0x1000
    arr = lambda *v: (P * len(v))(*[P(x) if x else None for x in v])  # noqa: E731
    ints = lambda *v: (ctypes.c_int * len(v))(*v)  # noqa: E731
    f = lib.tq_pack_shared_input
    ok_args = dict(n=2, Wq=arr(FAKE, FAKE), s_w=arr(FAKE, FAKE), L1t=arr(FAKE, FAKE),
                   L2t=arr(FAKE, FAKE), N=ints(64, 64), r=ints(16, 16), K=256)

    def call(**k):
        a = dict(ok_args, **k)
        return f(a["n"], a["Wq"], a["s_w"], a["L1t"], a["L2t"], a["N"], a["r"], a["K"], P(FAKE),
                 P(FAKE), P(FAKE), P(FAKE), None)
    assert call(n=0) == 1                         # no projection
    assert call(n=9) == 1                         # more than 8
    assert call(N=ints(64, 60)) == 2              # N % 8
    assert call(r=ints(16, 24)) == 2              # r % 16
    assert call(r=ints(256, 272)) == 2            # sum r > 512
    assert call(K=200) == 2
    assert call(L1t=arr(FAKE, 0)) == 1            # r > 0 needs L1^T
    assert call(Wq=arr(FAKE, FAKE + 4)) == 3      # alignment
