"""The one-kernel decode layer (tq_w4a4_lr_layer at M <= 16) through its
debug hook, which also returns the codes, scales and integer sums the
kernel computed on the way:

* codes and scales against the oracle (midpoint rule; scales to 2e-6), and
  equal bit for bit to tq_quantize_act's (the same butterflies);
* the INT32 sums equal, bit for bit, the oracle's integer GEMM of the
  same codes: these activation codes and the packed weight codes the kernel
  read (both checked against the oracle's under the midpoint rule;
  TwinQuant notes section 04.C: the residual accumulates in INT32);
* Y against the oracle's fp64 Y at the layer tolerance, and at rank 0 bit
  for bit against bf16((s_w s_x) acc) evaluated in float32 on the host;
* the layer entry point gives the same Y as the hook, and is deterministic.
"""
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


CASES = [
    # name, M, K, N, r, b
    ("decode_m16_llama3", 16, 4096, 4096, 32, 128),
    ("decode_m1", 1, 4096, 4096, 32, 128),
    ("m3_rank16", 3, 4096, 1024, 16, 128),
    ("rank0_m16", 16, 4096, 4096, 0, 128),
    ("rank0_block16", 7, 2048, 520, 0, 16),
    ("one_cta_k256", 16, 256, 512, 32, 256),
    ("cluster12_k3072", 5, 3072, 1536, 32, 128),
    ("ragged_n136", 16, 1024, 136, 16, 64),
    ("block256", 9, 2048, 384, 32, 256),
    ("block2", 4, 1024, 256, 16, 2),
    ("no_rotation", 2, 1024, 128, 32, 1),
    ("wide_n", 16, 1024, 8192, 32, 128),
    # rank 64 (one CTA per SM)
    ("rank64_m16", 16, 4096, 4096, 64, 128),
    ("rank64_cluster8", 5, 2048, 1024, 64, 128),
    ("rank64_cluster4_ragged", 11, 1024, 136, 64, 64),
    ("rank64_m1_block256", 1, 2048, 640, 64, 256),
]


@pytest.mark.parametrize("name,M,K,N,r,b", CASES, ids=[c[0] for c in CASES])
def test_decode_kernel_against_oracle(tq, name, M, K, N, r, b):
    assert tq.tq_layer_path(M, N, K, r, b) == "fused"
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r, had_block=b)
    L = synth.make_layer(sh, seed=3, device="cuda" if K * N >= 1 << 22 else "cpu")
    X, Rt = L["X"].cuda(), L["Rt"].cuda()
    L1t = L["L1t"].cuda() if r else None
    L2t = L["L2t"].cuda() if r else None
    Wq, s_w = tq.tq_pack_weight(Rt, b)
    Y, codes, s_x, acc = tq.tq_debug_w4a4_lr_layer_decode(X, L1t, Wq, s_w, L2t, b)
    Y_entry = tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, b)
    Xq, s_x2, _ = tq.tq_quantize_act(X, b, L1t)
    torch.cuda.synchronize()
    o = oracle.layer(L["X"], L["L1t"], L["L2t"], L["Rt"], b)
    q = codes.cpu().numpy()
    fx = check_codes(q, o["qx"], o["t_x"], f"{name}: codes", packed=False)
    check_scales(s_x.cpu().numpy(), o["s_x"], f"{name}: s_x")
    # the same codes and scales as the activation kernel of the two-call path
    assert np.array_equal(q, oracle.unpack_int4(Xq.cpu().numpy())), name
    assert torch.equal(s_x, s_x2), name
    qw = oracle.unpack_int4(Wq.cpu().numpy())
    fw = check_codes(qw, o["qw"], o["t_w"], f"{name}: weight codes", packed=False)
    # INT32 sums: bit for bit the integer GEMM of the codes the kernel used
    want_acc = oracle.int_gemm(q, qw)
    got_acc = acc.cpu().numpy().astype(np.int64)
    assert np.array_equal(got_acc, want_acc), (name, int((got_acc != want_acc).sum()))
    y = Y.double().cpu().numpy()
    fro, mx = check_y(y, y_reference(q, o, fx, qw, fw), name)
    if r == 0:
        # the epilogue in float32, as the kernel evaluates it
        sx = s_x.cpu().numpy().astype(np.float32)
        sw = s_w.cpu().numpy().astype(np.float32)
        y32 = (sw[None, :] * sx[:, None]) * acc.cpu().numpy().astype(np.float32)
        want = torch.from_numpy(y32).to(torch.bfloat16)
        assert torch.equal(Y.cpu(), want), name
    assert torch.equal(Y, Y_entry), name
    print(f"FLIPS decode {name}: x={fx:.3e} w={fw:.3e} fro={fro:.3e} max={mx:.3e}")


def test_decode_kernel_deterministic_and_reentrant(tq):
    sh = synth.CONFIGS["decode"].with_(M=16, K=4096, N=2048, r=32)
    L = synth.make_layer(sh, seed=4, device="cuda")
    X, Rt, L1t, L2t = (L[k].cuda() for k in ("X", "Rt", "L1t", "L2t"))
    Wq, s_w = tq.tq_pack_weight(Rt, 128)
    ys = [tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128) for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(ys[0], y)


def test_decode_kernel_chain_of_layers(tq):
    """Layers launched back to back on one stream (the next layer's CTAs
    share the SMs with the current one's): each output equals the layer
    computed alone."""
    sh = synth.CONFIGS["decode"].with_(M=16, K=4096, N=4096, r=32)
    lays = []
    for i in range(6):
        L = synth.make_layer(sh, seed=20 + i, device="cuda")
        Wq, s_w = tq.tq_pack_weight(L["Rt"].cuda(), 128)
        lays.append((L["X"].cuda(), L["L1t"].cuda(), Wq, s_w, L["L2t"].cuda()))
    alone = []
    for X, L1t, Wq, s_w, L2t in lays:
        alone.append(tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128))
        torch.cuda.synchronize()
    chained = [tq.tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, 128) for X, L1t, Wq, s_w, L2t in lays]
    torch.cuda.synchronize()
    for a, c in zip(alone, chained):
        assert torch.equal(a, c)
