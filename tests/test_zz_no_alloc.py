"""The allocation-free GEMM entry point, for callers that cannot call
cudaMalloc (for instance code inside a framework that owns the device
allocator, or a path that must not synchronise the device by allocating).

tq_w4a4_lr_gemm_noalloc takes the same inputs and output as tq_w4a4_lr_gemm
but no workspace: its scratch is a fixed array inside the library.  This
file checks, through the C ABI, that two calls in a row give the result of
the entry point with a caller workspace, within the layer's output tolerance.
It is collected last so that a run stopping at the first failure has run
every other test already; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from tests.parity_util import check_y

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
    y_ref = ref.double().cpu().numpy()
    for _ in range(2):  # the scratch keeps the previous call's contents
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        tq.tq_w4a4_lr_gemm_noalloc(Xq, s_x, Wq, s_w, XL1, L2t, Y=out)
        torch.cuda.synchronize()
        y = out.double().cpu().numpy()
        assert np.isfinite(y).all()
        check_y(y, y_ref, "noalloc vs workspace entry")
