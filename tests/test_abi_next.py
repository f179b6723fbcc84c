"""Host-side checks of the C ABI entry points of the NEXT rows built (shared-
input gate/up pair, asymmetric activations, INT4 low-rank branch) and of the
one-code-per-byte pair: bad arguments are rejected before any launch, and on
a machine without a GPU valid-looking arguments stop at the device check.
No compute call is made here."""
import ctypes

import pytest
import torch

P = ctypes.c_void_p
FAKE = 0x1000  # never dereferenced: every call below fails validation first
MIS = FAKE + 8  # not 16-byte aligned
OK, INVALID, SHAPE, MISALIGNED, WORKSPACE, NO_DEVICE = 0, 1, 2, 3, 6, 7
BIG = 1 << 40

no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")


@pytest.fixture(scope="module")
def lib():
    import rank_int4_gemm_b200 as tq
    return tq.tq.raw()


def _p(v):
    return None if v is None else P(v)


# ------------------------------------------------------- codes one per byte

def test_quantize_act_i8_validation(lib):
    def f(X=FAKE, M=4, K=512, b=128, L1t=None, r=0, Xq8=FAKE, s_x=FAKE, XL1b=None):
        return lib.tq_quantize_act_i8(_p(X), M, K, b, _p(L1t), r, _p(Xq8), _p(s_x), _p(XL1b), None)
    assert f(X=None) == INVALID
    assert f(M=0) == INVALID
    assert f(K=200) == SHAPE
    assert f(b=256) == SHAPE                       # tensor-core kernel: blocks up to 128
    assert f(r=16) == INVALID                      # r > 0 needs L1t and XL1b
    assert f(L1t=FAKE, r=16) == INVALID
    assert f(r=24, L1t=FAKE, XL1b=FAKE) == SHAPE   # r % 16
    assert f(X=MIS) == MISALIGNED
    assert f(r=16, L1t=FAKE, XL1b=MIS) == MISALIGNED


def test_gemm_a8_validation(lib):
    def f(Xq8=FAKE, XL1b=None, L2t=None, M=4, N=64, K=256, r=0, Y=FAKE, ws=FAKE, wsb=BIG):
        return lib.tq_w4a4_lr_gemm_a8(_p(Xq8), P(FAKE), P(FAKE), P(FAKE), _p(XL1b), _p(L2t), M, N,
                                      K, r, _p(Y), _p(ws), wsb, None)
    assert f(Y=None) == INVALID
    assert f(N=12) == SHAPE
    assert f(N=4) == SHAPE
    assert f(K=200) == SHAPE
    assert f(r=16) == INVALID
    assert f(r=16, XL1b=FAKE, L2t=MIS) == MISALIGNED
    assert f(ws=None) == WORKSPACE
    assert f(wsb=16) == WORKSPACE


# ------------------------------------------------------------- gate / up

def test_pack_gate_up_validation(lib):
    def f(r=0, lr=None, N=64, K=256, Wq2=FAKE):
        L = [lr] * 6 if lr is not None else [None] * 6
        return lib.tq_pack_gate_up(P(FAKE), P(FAKE), _p(L[0]), _p(L[1]), P(FAKE), P(FAKE),
                                   _p(L[2]), _p(L[3]), N, K, r, _p(Wq2), P(FAKE), _p(L[4]),
                                   _p(L[5]), None)
    assert f(N=0) == INVALID
    assert f(K=100) == SHAPE
    assert f(r=272, lr=FAKE) == SHAPE            # the stacked rank 2r must stay <= 512
    assert f(r=16) == INVALID                    # r > 0 needs every low-rank factor
    assert f(r=0, lr=FAKE) == INVALID            # r = 0 takes none
    assert f(Wq2=MIS) == MISALIGNED


def test_gate_up_validation(lib):
    def f(X=FAKE, L=None, M=4, N=64, K=512, r2=0, b=128, ws=FAKE, wsb=BIG):
        return lib.tq_w4a4_lr_gate_up(_p(X), _p(L), P(FAKE), P(FAKE), _p(L), M, N, K, r2, b,
                                      P(FAKE), _p(ws), wsb, None)
    assert f(X=None) == INVALID
    assert f(b=256) == SHAPE
    assert f(N=12) == SHAPE
    assert f(r2=48, L=FAKE) == SHAPE             # stacked rank: a multiple of 32
    assert f(r2=32) == INVALID                   # r2 > 0 needs L1t2 and L2t2
    assert f(X=MIS) == MISALIGNED
    assert f(ws=None) == WORKSPACE
    assert f(wsb=16) == WORKSPACE


def test_gate_up_workspace_grows_with_the_shape(lib):
    w = lib.tq_gate_up_workspace_bytes
    base = w(128, 64, 512, 32)
    assert base >= 256 + 128 * 512 + 128 * 4 + 128 * 32 * 2
    assert w(256, 64, 512, 32) > base and w(128, 64, 1024, 32) > base and w(128, 64, 512, 64) > base


# ---------------------------------------------------- asymmetric activations

def test_weight_code_sums_validation(lib):
    f = lib.tq_weight_code_sums
    assert f(None, 8, 256, P(FAKE), None) == INVALID
    assert f(P(FAKE), 0, 256, P(FAKE), None) == INVALID
    assert f(P(FAKE), 8, 100, P(FAKE), None) == SHAPE
    assert f(P(MIS), 8, 256, P(FAKE), None) == MISALIGNED


def test_quantize_act_asym_validation(lib):
    def f(z_x=FAKE, b=128, L1t=None, r=0, XL1b=None):
        return lib.tq_quantize_act_asym_i8(P(FAKE), 4, 512, b, _p(L1t), r, P(FAKE), P(FAKE),
                                           _p(z_x), _p(XL1b), None)
    assert f(z_x=None) == INVALID
    assert f(b=256) == SHAPE
    assert f(r=16, L1t=FAKE) == INVALID
    assert f(z_x=MIS) == MISALIGNED


def test_gemm_a8_asym_validation(lib):
    def f(wsum=FAKE, N=64, ws=FAKE, wsb=BIG, r=0, XL1b=None, L2t=None):
        return lib.tq_w4a4_lr_gemm_a8_asym(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), _p(wsum),
                                           _p(XL1b), _p(L2t), 4, N, 256, r, P(FAKE), _p(ws), wsb,
                                           None)
    assert f(wsum=None) == INVALID
    assert f(N=12) == SHAPE
    assert f(r=16, XL1b=FAKE) == INVALID
    assert f(wsum=MIS) == MISALIGNED
    assert f(wsb=16) == WORKSPACE


# ---------------------------------------------------- INT4 low-rank branch

def test_pack_lowrank_q4_validation(lib):
    def f(r=16, K=256, b=128, qL1=FAKE, L2t=FAKE):
        return lib.tq_pack_lowrank_q4(P(FAKE), _p(L2t), 64, K, r, b, _p(qL1), P(FAKE), P(FAKE),
                                      P(FAKE), None)
    assert f(r=0) == INVALID                     # the branch needs a rank
    assert f(L2t=None) == INVALID
    assert f(r=24) == SHAPE
    assert f(r=528) == SHAPE
    assert f(K=384, b=256) == SHAPE              # block does not divide K
    assert f(qL1=MIS) == MISALIGNED


def test_quantize_act_qlr_validation(lib):
    need = lib.tq_quantize_act_qlr_workspace_bytes(64, 512, 32)
    assert need >= 256 + 64 * 32 * 4             # status word + INT32 sums for wide ranks

    def f(r=32, b=128, XL1q=FAKE, ws=FAKE, wsb=BIG, qL1=FAKE):
        return lib.tq_quantize_act_qlr_i8(P(FAKE), 64, 512, b, _p(qL1), P(FAKE), r, P(FAKE),
                                          P(FAKE), _p(XL1q), P(FAKE), _p(ws), wsb, None)
    assert f(r=0) == INVALID
    assert f(qL1=None) == INVALID
    assert f(b=256) == SHAPE
    assert f(r=40) == SHAPE
    assert f(XL1q=MIS) == MISALIGNED
    assert f(ws=None) == WORKSPACE
    assert f(wsb=need - 1) == WORKSPACE


def test_gemm_a8_qlr_validation(lib):
    def f(s_L2=FAKE, r=32, N=64, ws=FAKE, wsb=BIG, qL2=FAKE):
        return lib.tq_w4a4_lr_gemm_a8_qlr(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                                          _p(qL2), _p(s_L2), 4, N, 256, r, P(FAKE), _p(ws), wsb,
                                          None)
    assert f(s_L2=None) == INVALID
    assert f(r=0) == INVALID
    assert f(N=12) == SHAPE
    assert f(qL2=MIS) == MISALIGNED
    assert f(wsb=16) == WORKSPACE


# ------------------------------------------------------ no device, no launch

@no_gpu
def test_valid_calls_stop_at_the_device_check(lib):
    """Arguments that pass every check reach the device check, which fails
    here (no GPU), so nothing is launched."""
    assert lib.tq_quantize_act_i8(P(FAKE), 4, 512, 128, None, 0, P(FAKE), P(FAKE), None,
                                  None) == NO_DEVICE
    assert lib.tq_pack_lowrank_q4(P(FAKE), P(FAKE), 64, 256, 16, 128, P(FAKE), P(FAKE), P(FAKE),
                                  P(FAKE), None) == NO_DEVICE
    assert lib.tq_quantize_act_qlr_i8(P(FAKE), 64, 512, 128, P(FAKE), P(FAKE), 32, P(FAKE),
                                      P(FAKE), P(FAKE), P(FAKE), P(FAKE), BIG, None) == NO_DEVICE
    assert lib.tq_weight_code_sums(P(FAKE), 8, 256, P(FAKE), None) == NO_DEVICE
    assert lib.tq_w4a4_lr_gate_up(P(FAKE), None, P(FAKE), P(FAKE), None, 4, 64, 512, 0, 128,
                                  P(FAKE), P(FAKE), BIG, None) == NO_DEVICE
