"""The allocation-free GEMM entry point, for callers that cannot call
cudaMalloc (for instance code inside a framework that owns the device
allocator, or a path that must not synchronise the device by allocating).

tq_w4a4_lr_gemm_noalloc takes the same inputs and output as tq_w4a4_lr_gemm
but no workspace: its scratch is a fixed array inside the library.  This
file checks, through the C ABI, that two calls in a row give exactly the
result of the entry point with a caller workspace (the same kernel on the
same inputs), and that the scratch's status word is read and cleared by
tq_noalloc_query_status.  It is collected last so that a run stopping at the
first failure has run every other test already; it also passes on its own in
a fresh process.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

CASES = [
    # M, K, N, r: the decode tiling (split-K cluster) and the prefill tiling
    (16, 1024, 512, 32),
    (200, 512, 264, 16),
]


@pytest.mark.parametrize("M,K,N,r", CASES)
def test_noalloc_matches_workspace_entry(cuda_ok, M, K, N, r):
    import rank_int4_gemm_b200 as tq
    sh = synth.CONFIGS["decode"].with_(M=M, K=K, N=N, r=r)
    L = synth.make_layer(sh)
    X, L1t, L2t, Rt = (L[k].contiguous().cuda() for k in ("X", "L1t", "L2t", "Rt"))
    Wq, s_w = tq.tq_pack_weight(Rt, sh.had_block)
    Xq, s_x, XL1 = tq.tq_quantize_act(X, sh.had_block, L1t)
    ref = tq.tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t)
    torch.cuda.synchronize()
    for _ in range(2):  # the scratch keeps the previous call's contents
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        tq.tq_w4a4_lr_gemm_noalloc(Xq, s_x, Wq, s_w, XL1, L2t, Y=out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert tq.tq_noalloc_query_status() == 0


def test_noalloc_status_word_read_and_cleared(cuda_ok):
    import rank_int4_gemm_b200 as tq
    assert tq.tq_noalloc_query_status() == 0
    tq.tq_debug_noalloc_set_status(5)           # what a wait that gave up writes
    assert tq.tq_noalloc_query_status() == 5    # TQ_ERR_TIMEOUT, reported once
    assert tq.tq_noalloc_query_status() == 0    # and cleared by the query


def test_noalloc_argument_errors_before_device_work(cuda_ok):
    import ctypes

    import rank_int4_gemm_b200 as tq
    lib = tq.tq.raw()
    P = ctypes.c_void_p
    Xq = torch.zeros(16, 256, dtype=torch.uint8, device="cuda")
    Wq = torch.zeros(128, 256, dtype=torch.uint8, device="cuda")
    s = torch.zeros(128, dtype=torch.float32, device="cuda")
    Y = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    p = lambda t: P(t.data_ptr())  # noqa: E731
    # r > 0 without X L1 / L2^T: invalid value, nothing launched
    assert lib.tq_w4a4_lr_gemm_noalloc(p(Xq), p(s), p(Wq), p(s), None, None, 16, 128, 512, 16,
                                       p(Y), None) == 1
    # K not a multiple of 128: unsupported shape
    assert lib.tq_w4a4_lr_gemm_noalloc(p(Xq), p(s), p(Wq), p(s), None, None, 16, 128, 500, 0,
                                       p(Y), None) == 2
    torch.cuda.synchronize()
    assert tq.tq_noalloc_query_status() == 0
