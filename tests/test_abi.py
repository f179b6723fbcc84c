"""Host-side checks of the C ABI: the library loads, exports every entry
point include/tq.h declares, and rejects bad arguments before any launch.
No compute call is made here (runs without a GPU)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tq.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import rank_int4_gemm_b200 as tq
    return tq.tq.raw()


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("tq_pack_weight", "tq_quantize_act", "tq_w4a4_lr_gemm", "tq_gemm_workspace_bytes",
              "tq_debug_w4a4_gemm_acc", "tq_query_device_status", "tq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in _declared():
        assert hasattr(lib, n), n


def test_status_strings(lib):
    import rank_int4_gemm_b200 as tq
    assert tq.tq_status_string(0) == "TQ_OK"
    assert tq.tq_status_string(5) == "TQ_ERR_TIMEOUT"
    assert tq.tq_status_string(99) == "TQ_ERR_UNKNOWN"
    assert tq.tq_version() >= 100


P = ctypes.c_void_p
FAKE = 0x1000  # never dereferenced: every call below fails validation first


def test_pack_weight_validation(lib):
    assert lib.tq_pack_weight(None, 8, 128, 128, P(FAKE), P(FAKE), None) == 1
    assert lib.tq_pack_weight(P(FAKE), 0, 128, 128, P(FAKE), P(FAKE), None) == 1
    assert lib.tq_pack_weight(P(FAKE), 8, 100, 128, P(FAKE), P(FAKE), None) == 2
    assert lib.tq_pack_weight(P(FAKE), 8, 384, 256, P(FAKE), P(FAKE), None) == 2   # b !| K
    assert lib.tq_pack_weight(P(FAKE), 8, 256, 96, P(FAKE), P(FAKE), None) == 2    # b not 2^k
    assert lib.tq_pack_weight(P(FAKE), 8, 256, 512, P(FAKE), P(FAKE), None) == 2   # b > 256
    assert lib.tq_pack_weight(P(FAKE), 8, 65536, 128, P(FAKE), P(FAKE), None) == 2  # K too big
    assert lib.tq_pack_weight(P(FAKE + 4), 8, 256, 128, P(FAKE), P(FAKE), None) == 3


def test_quantize_act_validation(lib):
    f = lib.tq_quantize_act
    assert f(None, 4, 256, 128, None, 0, P(FAKE), P(FAKE), None, None) == 1
    assert f(P(FAKE), 4, 256, 128, None, 16, P(FAKE), P(FAKE), P(FAKE), None) == 1  # r>0, no L1
    assert f(P(FAKE), 4, 256, 128, P(FAKE), 0, P(FAKE), P(FAKE), None, None) == 1   # L1, r=0
    assert f(P(FAKE), 4, 256, 128, P(FAKE), 24, P(FAKE), P(FAKE), P(FAKE), None) == 2  # r%16
    assert f(P(FAKE), 4, 256, 128, P(FAKE), 528, P(FAKE), P(FAKE), P(FAKE), None) == 2  # r>512
    assert f(P(FAKE), 4, 256, 128, None, 0, P(FAKE + 8), P(FAKE), None, None) == 3


def test_gemm_validation(lib):
    f = lib.tq_w4a4_lr_gemm
    args = lambda **k: [k.get("Xq", P(FAKE)), P(FAKE), P(FAKE), P(FAKE), k.get("XL1"),
                        k.get("L2t"), k.get("M", 4), k.get("N", 64), k.get("K", 256),
                        k.get("r", 0), k.get("Y", P(FAKE)), k.get("ws", P(FAKE)),
                        ctypes.c_size_t(k.get("wsb", 1 << 30)), None]
    assert f(*args(Y=None)) == 1
    assert f(*args(N=60)) == 2
    assert f(*args(N=4)) == 2
    assert f(*args(K=200)) == 2
    assert f(*args(r=16)) == 1                          # r > 0 needs XL1 and L2t
    assert f(*args(r=16, XL1=P(FAKE), L2t=P(FAKE + 2))) == 3
    assert f(*args(ws=None)) == 6
    assert f(*args(wsb=16)) == 6
    assert lib.tq_gemm_workspace_bytes(1, 4096, 4096, 32) >= 256


def test_noalloc_validation(lib):
    # the no-allocation entry checks its arguments before any device work
    f = lib.tq_w4a4_lr_gemm_noalloc
    args = lambda **k: [k.get("Xq", P(FAKE)), P(FAKE), P(FAKE), P(FAKE), k.get("XL1"),
                        k.get("L2t"), k.get("M", 4), k.get("N", 64), k.get("K", 256),
                        k.get("r", 0), k.get("Y", P(FAKE)), None]
    assert f(*args(Y=None)) == 1
    assert f(*args(Xq=None)) == 1
    assert f(*args(N=60)) == 2
    assert f(*args(K=200)) == 2
    assert f(*args(r=16)) == 1
    assert f(*args(r=16, XL1=P(FAKE), L2t=P(FAKE + 2))) == 3


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_no_device_is_reported(lib):
    # Valid-looking arguments pass validation, then the device check fails
    # (this container has no GPU), so nothing is launched.
    assert lib.tq_pack_weight(P(FAKE), 8, 256, 128, P(FAKE), P(FAKE), None) == 7


def test_layer_path_routing():
    """tq_layer_path is a host query (runs without a GPU): the one-kernel
    decode layer where its limits hold (M <= 16, r in {0, 16, 32, 64}, K % 256 == 0,
    K <= 4096, Hadamard block <= 256), int8 codes for M > 128 with block
    <= 128, packed codes otherwise; rejected shapes raise."""
    import rank_int4_gemm_b200 as tq
    p = tq.tq_layer_path
    assert p(16, 4096, 4096, 32, 128) == "fused"
    assert p(1, 4096, 4096, 0, 128) == "fused"
    assert p(16, 4096, 4096, 32, 1) == "fused"
    assert p(17, 4096, 4096, 32, 128) == "codes_packed"
    assert p(16, 4096, 4096, 64, 128) == "fused"
    assert p(16, 4096, 4096, 48, 128) == "codes_packed"   # ranks 0, 16, 32, 64 only
    assert p(16, 4096, 3840, 64, 128) == "codes_packed"   # rank 64: clusters dividing 16
    assert p(16, 4096, 3840, 32, 128) == "fused"
    assert p(16, 8192, 4096, 32, 128) == "fused"        # N does not limit it
    assert p(16, 4096, 4608, 32, 128) == "codes_packed"  # K > 4096
    assert p(16, 4096, 384, 16, 128) == "codes_packed"   # K % 256 != 0
    assert p(16, 4096, 768, 16, 128) == "fused"          # a cluster of 3 CTAs
    assert p(16, 4096, 4096, 32, 256) == "fused"
    assert p(128, 4096, 4096, 64, 128) == "codes_packed"
    assert p(129, 4096, 4096, 64, 128) == "codes_i8"
    assert p(4096, 4096, 4096, 128, 128) == "codes_i8"
    assert p(4096, 4096, 4096, 512, 128) == "codes_i8"
    assert p(4096, 4096, 4096, 64, 256) == "codes_packed"
    for bad in [(0, 4096, 4096, 32, 128), (16, 4096, 4000, 32, 128), (16, 4096, 4096, 24, 128),
                (16, 12, 4096, 32, 128)]:
        with pytest.raises(tq.TQError):
            p(*bad)
