"""ctypes binding of libtq.so: argument marshalling only.

Every function has the name of the C entry point it calls and forwards torch
tensors as raw device pointers plus the current CUDA stream.  Outputs that the
caller does not pass are allocated with torch (plumbing); nothing is computed
here.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libtq.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python rank_int4_gemm_b200/build_lib.py` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(_LIB_PATH)
_P = ctypes.c_void_p
_I = ctypes.c_int

_lib.tq_status_string.restype = ctypes.c_char_p
_lib.tq_status_string.argtypes = [_I]
_lib.tq_version.restype = _I
_lib.tq_pack_weight.restype = _I
_lib.tq_pack_weight.argtypes = [_P, _I, _I, _I, _P, _P, _P]
_lib.tq_quantize_act.restype = _I
_lib.tq_quantize_act.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P, _P, _P]
_lib.tq_gemm_workspace_bytes.restype = ctypes.c_size_t
_lib.tq_gemm_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.tq_gemm_a8_workspace_bytes.restype = ctypes.c_size_t
_lib.tq_gemm_a8_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.tq_w4a4_lr_gemm.restype = _I
_lib.tq_w4a4_lr_gemm.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P,
                                  ctypes.c_size_t, _P]
_lib.tq_debug_w4a4_gemm_acc.restype = _I
_lib.tq_debug_w4a4_gemm_acc.argtypes = [_P, _P, _I, _I, _I, _P, _P, ctypes.c_size_t, _P]
_lib.tq_w4a4_lr_gemm_noalloc.restype = _I
_lib.tq_w4a4_lr_gemm_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P]
_lib.tq_pack_weight_rht.restype = _I
_lib.tq_pack_weight_rht.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P]
_lib.tq_quantize_act_rht.restype = _I
_lib.tq_quantize_act_rht.argtypes = [_P, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P]
_lib.tq_w4a4_lr_layer_rht.restype = _I
_lib.tq_w4a4_lr_layer_rht.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P,
                                      ctypes.c_size_t, _P]
_lib.tq_pack_weight_rhtn.restype = _I
_lib.tq_pack_weight_rhtn.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P, _P]
_lib.tq_quantize_act_rhtn.restype = _I
_lib.tq_quantize_act_rhtn.argtypes = [_P, _I, _I, _I, _P, _I, _P, _I, _P, _P, _P, _P]
_lib.tq_w4a4_lr_layer_rhtn.restype = _I
_lib.tq_w4a4_lr_layer_rhtn.argtypes = [_P, _P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P,
                                       ctypes.c_size_t, _P]
_lib.tq_pack_shared_input.restype = _I
_lib.tq_pack_shared_input.argtypes = [_I, _P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P]
_lib.tq_debug_w4a4_lr_layer_decode.restype = _I
_lib.tq_debug_w4a4_lr_layer_decode.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P,
                                               _P, _P, _P, ctypes.c_size_t, _P]
_lib.tq_debug_watchdog.restype = _I
_lib.tq_debug_watchdog.argtypes = [_P, ctypes.c_size_t, _I, ctypes.c_longlong, _P, _P]
_lib.tq_noalloc_query_status.restype = _I
_lib.tq_noalloc_query_status.argtypes = [_P]
_lib.tq_debug_noalloc_set_status.restype = _I
_lib.tq_debug_noalloc_set_status.argtypes = [_I]
_lib.tq_layer_workspace_bytes.restype = ctypes.c_size_t
_lib.tq_layer_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.tq_layer_path.restype = _I
_lib.tq_pack_lowrank_q4.restype = _I
_lib.tq_pack_lowrank_q4.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P]
_lib.tq_quantize_act_qlr_workspace_bytes.restype = ctypes.c_size_t
_lib.tq_quantize_act_qlr_workspace_bytes.argtypes = [_I, _I, _I]
_lib.tq_quantize_act_qlr_i8.restype = _I
_lib.tq_quantize_act_qlr_i8.argtypes = [_P, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]
_lib.tq_w4a4_lr_gemm_a8_qlr.restype = _I
_lib.tq_w4a4_lr_gemm_a8_qlr.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P,
                                        _P, ctypes.c_size_t, _P]
_lib.tq_quantize_act_asym_i8.restype = _I
_lib.tq_quantize_act_asym_i8.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P]
_lib.tq_weight_code_sums.restype = _I
_lib.tq_weight_code_sums.argtypes = [_P, _I, _I, _P, _P]
_lib.tq_w4a4_lr_gemm_a8_asym.restype = _I
_lib.tq_w4a4_lr_gemm_a8_asym.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P,
                                         _P, ctypes.c_size_t, _P]
_lib.tq_pack_gate_up.restype = _I
_lib.tq_pack_gate_up.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P, _P]
_lib.tq_gate_up_workspace_bytes.restype = ctypes.c_size_t
_lib.tq_gate_up_workspace_bytes.argtypes = [_I, _I, _I, _I]
_lib.tq_w4a4_lr_gate_up.restype = _I
_lib.tq_w4a4_lr_gate_up.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P,
                                    ctypes.c_size_t, _P]
_lib.tq_layer_path.argtypes = [_I, _I, _I, _I, _I]
_lib.tq_w4a4_lr_layer.restype = _I
_lib.tq_w4a4_lr_layer.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P,
                                  ctypes.c_size_t, _P]
_lib.tq_quantize_act_i8.restype = _I
_lib.tq_quantize_act_i8.argtypes = [_P, _I, _I, _I, _P, _I, _P, _P, _P, _P]
_lib.tq_w4a4_lr_gemm_a8.restype = _I
_lib.tq_w4a4_lr_gemm_a8.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P,
                                    ctypes.c_size_t, _P]
_lib.tq_query_device_status.restype = _I
_lib.tq_query_device_status.argtypes = [_P, _P]


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {tq_status_string(status)} ({status})")


def lib_path() -> str:
    return _LIB_PATH


def raw() -> ctypes.CDLL:
    """The loaded C library (for callers passing raw pointers)."""
    return _lib


def tq_status_string(status: int) -> str:
    return _lib.tq_status_string(int(status)).decode()


def tq_version() -> int:
    return int(_lib.tq_version())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int, where: str):
    if st != 0:
        raise TQError(st, where)


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def tq_pack_weight(Rt: torch.Tensor, had_block: int, Wq=None, s_w=None, stream=None):
    """R^T [N][K] fp32 -> (Wq [N][K/2] uint8, s_w [N] fp32)."""
    N, K = Rt.shape
    _need(Rt, torch.float32, (N, K), "Rt")
    if Wq is None:
        Wq = torch.empty(N, K // 2, dtype=torch.uint8, device=Rt.device)
    if s_w is None:
        s_w = torch.empty(N, dtype=torch.float32, device=Rt.device)
    _check(_lib.tq_pack_weight(_ptr(Rt), N, K, int(had_block), _ptr(Wq), _ptr(s_w),
                               _stream(stream)), "tq_pack_weight")
    return Wq, s_w


def tq_quantize_act(X: torch.Tensor, had_block: int, L1t=None, Xq=None, s_x=None, XL1=None,
                    stream=None):
    """X [M][K] bf16 (+ L1^T [r][K] bf16) -> (Xq [M][K/2] u8, s_x [M] f32, XL1 [M][r] f32)."""
    M, K = X.shape
    _need(X, torch.bfloat16, (M, K), "X")
    r = 0 if L1t is None else L1t.shape[0]
    if r:
        _need(L1t, torch.bfloat16, (r, K), "L1t")
    dev = X.device
    if Xq is None:
        Xq = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
    if s_x is None:
        s_x = torch.empty(M, dtype=torch.float32, device=dev)
    if r and XL1 is None:
        XL1 = torch.empty(M, r, dtype=torch.float32, device=dev)
    _check(_lib.tq_quantize_act(_ptr(X), M, K, int(had_block), _ptr(L1t) if r else None, r,
                                _ptr(Xq), _ptr(s_x), _ptr(XL1) if r else None, _stream(stream)),
           "tq_quantize_act")
    return Xq, s_x, (XL1 if r else None)


def tq_quantize_act_i8(X: torch.Tensor, had_block: int, L1t=None, Xq8=None, s_x=None, XL1b=None,
                       stream=None):
    """X [M][K] bf16 (+ L1^T) -> (Xq8 [M][K] int8 codes, s_x [M] f32, XL1b [M][r] bf16)."""
    M, K = X.shape
    _need(X, torch.bfloat16, (M, K), "X")
    r = 0 if L1t is None else L1t.shape[0]
    if r:
        _need(L1t, torch.bfloat16, (r, K), "L1t")
    dev = X.device
    if Xq8 is None:
        Xq8 = torch.empty(M, K, dtype=torch.int8, device=dev)
    if s_x is None:
        s_x = torch.empty(M, dtype=torch.float32, device=dev)
    if r and XL1b is None:
        XL1b = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    _check(_lib.tq_quantize_act_i8(_ptr(X), M, K, int(had_block), _ptr(L1t) if r else None, r,
                                   _ptr(Xq8), _ptr(s_x), _ptr(XL1b) if r else None,
                                   _stream(stream)),
           "tq_quantize_act_i8")
    return Xq8, s_x, (XL1b if r else None)


def tq_gemm_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(_lib.tq_gemm_workspace_bytes(M, N, K, r))


def tq_gemm_a8_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    """Workspace of the codes-one-per-byte GEMMs with their stream-K scratch."""
    return int(_lib.tq_gemm_a8_workspace_bytes(M, N, K, r))


class Workspace:
    """A zero-filled device workspace that grows on demand (plumbing)."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


def tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1=None, L2t=None, Y=None, workspace=None,
                    stream=None):
    """Y [M][N] bf16 = s_x s_w (Xq . Wq) + bf16(XL1) L2^T."""
    M, K2 = Xq.shape
    N = Wq.shape[0]
    K = 2 * K2
    r = 0 if XL1 is None else XL1.shape[1]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xq.device)
    if workspace is None:
        workspace = Workspace(Xq.device)
    need = tq_gemm_workspace_bytes(M, N, K, r)
    ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    _check(_lib.tq_w4a4_lr_gemm(_ptr(Xq), _ptr(s_x), _ptr(Wq), _ptr(s_w),
                                _ptr(XL1) if r else None, _ptr(L2t) if r else None,
                                M, N, K, r, _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)),
           "tq_w4a4_lr_gemm")
    return Y


def tq_w4a4_lr_gemm_a8(Xq8, s_x, Wq, s_w, XL1b=None, L2t=None, Y=None, workspace=None,
                       stream=None):
    """Y [M][N] bf16 = s_x s_w (Xq8 . Wq) + XL1b L2^T, codes one per byte."""
    M, K = Xq8.shape
    N = Wq.shape[0]
    r = 0 if XL1b is None else XL1b.shape[1]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xq8.device)
    if workspace is None:
        workspace = Workspace(Xq8.device)
    need = tq_gemm_a8_workspace_bytes(M, N, K, r)
    ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    _check(_lib.tq_w4a4_lr_gemm_a8(_ptr(Xq8), _ptr(s_x), _ptr(Wq), _ptr(s_w),
                                   _ptr(XL1b) if r else None, _ptr(L2t) if r else None,
                                   M, N, K, r, _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)),
           "tq_w4a4_lr_gemm_a8")
    return Y


def tq_quantize_act_asym_i8(X: torch.Tensor, had_block: int, L1t=None, stream=None):
    """Per-token asymmetric codes: X [M][K] bf16 (+ L1^T) -> (Xq8 [M][K] int8
    = code - 8, s_x [M], z_x [M] f32, XL1b [M][r] bf16)."""
    M, K = X.shape
    _need(X, torch.bfloat16, (M, K), "X")
    r = 0 if L1t is None else L1t.shape[0]
    if r:
        _need(L1t, torch.bfloat16, (r, K), "L1t")
    dev = X.device
    Xq8 = torch.empty(M, K, dtype=torch.int8, device=dev)
    s_x = torch.empty(M, dtype=torch.float32, device=dev)
    z_x = torch.empty(M, dtype=torch.float32, device=dev)
    XL1b = torch.empty(M, r, dtype=torch.bfloat16, device=dev) if r else None
    _check(_lib.tq_quantize_act_asym_i8(_ptr(X), M, K, int(had_block), _ptr(L1t) if r else None,
                                        r, _ptr(Xq8), _ptr(s_x), _ptr(z_x),
                                        _ptr(XL1b) if r else None, _stream(stream)),
           "tq_quantize_act_asym_i8")
    return Xq8, s_x, z_x, XL1b


def tq_weight_code_sums(Wq, stream=None):
    """wsum [N] int32: the sum of each channel's weight codes."""
    N, K2 = Wq.shape
    wsum = torch.empty(N, dtype=torch.int32, device=Wq.device)
    _check(_lib.tq_weight_code_sums(_ptr(Wq), N, 2 * K2, _ptr(wsum), _stream(stream)),
           "tq_weight_code_sums")
    return wsum


def tq_w4a4_lr_gemm_a8_asym(Xq8, s_x, z_x, Wq, s_w, wsum, XL1b=None, L2t=None, Y=None,
                            workspace=None, stream=None):
    """Y [M][N] bf16 = s_w (s_x (acc + 8 wsum) + z_x wsum) + XL1b L2^T."""
    M, K = Xq8.shape
    N = Wq.shape[0]
    r = 0 if XL1b is None else XL1b.shape[1]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xq8.device)
    if workspace is None:
        workspace = Workspace(Xq8.device)
    need = tq_gemm_a8_workspace_bytes(M, N, K, r)
    ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    _check(_lib.tq_w4a4_lr_gemm_a8_asym(_ptr(Xq8), _ptr(s_x), _ptr(z_x), _ptr(Wq), _ptr(s_w),
                                        _ptr(wsum), _ptr(XL1b) if r else None,
                                        _ptr(L2t) if r else None, M, N, K, r, _ptr(Y), _ptr(ws),
                                        ws.numel(), _stream(stream)),
           "tq_w4a4_lr_gemm_a8_asym")
    return Y


def tq_pack_lowrank_q4(L1t, L2t, had_block, stream=None):
    """INT4 low-rank factors: (qL1 [r][K] s8 codes, s_L1 [r], qL2 [N][r] bf16
    integer codes, s_L2 [N])."""
    r, K = L1t.shape
    N = L2t.shape[0]
    dev = L1t.device
    qL1 = torch.empty(r, K, dtype=torch.int8, device=dev)
    s_L1 = torch.empty(r, dtype=torch.float32, device=dev)
    qL2 = torch.empty(N, r, dtype=torch.bfloat16, device=dev)
    s_L2 = torch.empty(N, dtype=torch.float32, device=dev)
    _check(_lib.tq_pack_lowrank_q4(_ptr(L1t), _ptr(L2t), N, K, r, int(had_block), _ptr(qL1),
                                   _ptr(s_L1), _ptr(qL2), _ptr(s_L2), _stream(stream)),
           "tq_pack_lowrank_q4")
    return qL1, s_L1, qL2, s_L2


def tq_quantize_act_qlr_i8(X, had_block, qL1, s_L1, workspace=None, stream=None):
    """(Xq8 [M][K] s8, s_x [M], XL1q [M][r] bf16 integer codes, s_xl1 [M])."""
    M, K = X.shape
    r = qL1.shape[0]
    dev = X.device
    Xq8 = torch.empty(M, K, dtype=torch.int8, device=dev)
    s_x = torch.empty(M, dtype=torch.float32, device=dev)
    XL1q = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    s_xl1 = torch.empty(M, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = Workspace(dev)
    need = int(_lib.tq_quantize_act_qlr_workspace_bytes(M, K, r))
    ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    _check(_lib.tq_quantize_act_qlr_i8(_ptr(X), M, K, int(had_block), _ptr(qL1), _ptr(s_L1), r,
                                       _ptr(Xq8), _ptr(s_x), _ptr(XL1q), _ptr(s_xl1), _ptr(ws),
                                       ws.numel(), _stream(stream)),
           "tq_quantize_act_qlr_i8")
    return Xq8, s_x, XL1q, s_xl1


def tq_w4a4_lr_gemm_a8_qlr(Xq8, s_x, Wq, s_w, XL1q, s_xl1, qL2, s_L2, Y=None, workspace=None,
                           stream=None):
    """Y [M][N] bf16 = s_x s_w (Xq8 . Wq) + s_xl1 s_L2 (XL1q . qL2)."""
    M, K = Xq8.shape
    N = Wq.shape[0]
    r = XL1q.shape[1]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xq8.device)
    if workspace is None:
        workspace = Workspace(Xq8.device)
    need = tq_gemm_a8_workspace_bytes(M, N, K, r)
    ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    _check(_lib.tq_w4a4_lr_gemm_a8_qlr(_ptr(Xq8), _ptr(s_x), _ptr(Wq), _ptr(s_w), _ptr(XL1q),
                                       _ptr(s_xl1), _ptr(qL2), _ptr(s_L2), M, N, K, r, _ptr(Y),
                                       _ptr(ws), ws.numel(), _stream(stream)),
           "tq_w4a4_lr_gemm_a8_qlr")
    return Y


def tq_w4a4_lr_gemm_noalloc(Xq, s_x, Wq, s_w, XL1=None, L2t=None, Y=None, stream=None):
    """tq_w4a4_lr_gemm without a workspace argument, for callers that cannot
    allocate device memory: the kernel's scratch is a fixed array inside the
    library (shared by all calls; overlapping calls race).  Y must be passed
    by such callers; it is allocated here only as a convenience."""
    M, K2 = Xq.shape
    N = Wq.shape[0]
    K = 2 * K2
    r = 0 if XL1 is None else XL1.shape[1]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=Xq.device)
    _check(_lib.tq_w4a4_lr_gemm_noalloc(_ptr(Xq), _ptr(s_x), _ptr(Wq), _ptr(s_w),
                                        _ptr(XL1) if r else None, _ptr(L2t) if r else None,
                                        M, N, K, r, _ptr(Y), _stream(stream)),
           "tq_w4a4_lr_gemm_noalloc")
    return Y


def tq_pack_shared_input(projections, stream=None):
    """Projections reading the same X, each (Wq, s_w, L1t, L2t) as
    tq_pack_weight makes them (L1t / L2t None for rank 0), packed as one
    layer: returns (Wq_cat, s_w_cat, L1t_cat, L2t_cat, N_list).  Run it with
    tq_w4a4_lr_layer; split_shared_output gives each projection's Y."""
    n = len(projections)
    Ns = [int(p[0].shape[0]) for p in projections]
    K = 2 * int(projections[0][0].shape[1])
    rs = [0 if p[2] is None else int(p[2].shape[0]) for p in projections]
    dev = projections[0][0].device
    n_cat, r_cat = sum(Ns), sum(rs)
    Wq_cat = torch.empty(n_cat, K // 2, dtype=torch.uint8, device=dev)
    s_w_cat = torch.empty(n_cat, dtype=torch.float32, device=dev)
    L1t_cat = torch.empty(r_cat, K, dtype=torch.bfloat16, device=dev) if r_cat else None
    L2t_cat = torch.empty(n_cat, r_cat, dtype=torch.bfloat16, device=dev) if r_cat else None
    arr = lambda ts: (ctypes.c_void_p * n)(*[None if t is None else t.data_ptr() for t in ts])  # noqa: E731
    _check(_lib.tq_pack_shared_input(
        n, arr([p[0] for p in projections]), arr([p[1] for p in projections]),
        arr([p[2] for p in projections]), arr([p[3] for p in projections]),
        (ctypes.c_int * n)(*Ns), (ctypes.c_int * n)(*rs), K, _ptr(Wq_cat), _ptr(s_w_cat),
        _ptr(L1t_cat), _ptr(L2t_cat), _stream(stream)), "tq_pack_shared_input")
    return Wq_cat, s_w_cat, L1t_cat, L2t_cat, Ns


def split_shared_output(Y, Ns):
    """Views of the concatenated layer's Y [M][sum N], one per projection."""
    return list(torch.split(Y, list(Ns), dim=1))


def tq_debug_w4a4_lr_layer_decode(X, L1t, Wq, s_w, L2t, had_block, workspace=None, stream=None):
    """The one-kernel decode layer with its debug outputs: returns
    (Y [M][N] bf16, codes [M][K] int8, s_x [M] fp32, acc [M][N] int32)."""
    M, K = X.shape
    N = Wq.shape[0]
    r = 0 if L1t is None else L1t.shape[0]
    dev = X.device
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    codes = torch.empty(M, K, dtype=torch.int8, device=dev)
    s_x = torch.empty(M, dtype=torch.float32, device=dev)
    acc = torch.empty(M, N, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = Workspace(dev)
    ws = workspace.get(256) if isinstance(workspace, Workspace) else workspace
    _check(_lib.tq_debug_w4a4_lr_layer_decode(_ptr(X), _ptr(L1t), _ptr(Wq), _ptr(s_w), _ptr(L2t),
                                              M, N, K, r, int(had_block), _ptr(Y), _ptr(codes),
                                              _ptr(s_x), _ptr(acc), _ptr(ws), ws.numel(),
                                              _stream(stream)),
           "tq_debug_w4a4_lr_layer_decode")
    return Y, codes, s_x, acc


def tq_debug_watchdog(workspace, withhold: bool, budget_cycles: int, waited_ok=None,
                      stream=None):
    """Test hook of the bounded waits: one CTA whose consumer waits (at most
    budget_cycles) for a producer arrival that `withhold` suppresses.
    Returns the device int set to 1 (arrival seen) or 0 (wait gave up)."""
    ws = workspace.get(256) if isinstance(workspace, Workspace) else workspace
    if waited_ok is None:
        waited_ok = torch.full((1,), -1, dtype=torch.int32, device=ws.device)
    _check(_lib.tq_debug_watchdog(_ptr(ws), ws.numel(), int(bool(withhold)), int(budget_cycles),
                                  _ptr(waited_ok), _stream(stream)), "tq_debug_watchdog")
    return waited_ok


def tq_noalloc_query_status(stream=None) -> int:
    """Status word of the no-allocation entry point's scratch (synchronises
    the stream, reads and clears it): 0, or 5 (TQ_ERR_TIMEOUT)."""
    return int(_lib.tq_noalloc_query_status(_stream(stream)))


def tq_debug_noalloc_set_status(status: int) -> None:
    """Test hook: write `status` into that word (synchronous, no kernel)."""
    _check(_lib.tq_debug_noalloc_set_status(int(status)), "tq_debug_noalloc_set_status")


def tq_debug_w4a4_gemm_acc(Xq, Wq, acc=None, workspace=None, stream=None):
    """Raw INT32 accumulators acc[m][n] = sum_k qx[m][k] qw[n][k]."""
    M, K2 = Xq.shape
    N = Wq.shape[0]
    K = 2 * K2
    if acc is None:
        acc = torch.empty(M, N, dtype=torch.int32, device=Xq.device)
    if workspace is None:
        workspace = Workspace(Xq.device)
    ws = workspace.get(tq_gemm_workspace_bytes(M, N, K, 0)) if isinstance(workspace, Workspace) \
        else workspace
    _check(_lib.tq_debug_w4a4_gemm_acc(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc), _ptr(ws),
                                       ws.numel(), _stream(stream)), "tq_debug_w4a4_gemm_acc")
    return acc


def tq_query_device_status(workspace, stream=None) -> int:
    ws = workspace.buf if isinstance(workspace, Workspace) else workspace
    return int(_lib.tq_query_device_status(_ptr(ws), _stream(stream)))


def tq_layer_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(_lib.tq_layer_workspace_bytes(M, N, K, r))


LAYER_PATHS = {0: "fused", 1: "codes_i8", 2: "codes_packed"}


def tq_layer_path(M: int, N: int, K: int, r: int, had_block: int) -> str:
    """Which kernels tq_w4a4_lr_layer runs for this shape (host query):
    "fused", "codes_i8" or "codes_packed"; raises on a shape it rejects."""
    v = int(_lib.tq_layer_path(M, N, K, r, had_block))
    if v < 0:
        raise TQError(-v, "tq_layer_path")
    return LAYER_PATHS[v]


def tq_w4a4_lr_layer(X, L1t, Wq, s_w, L2t, had_block, Y=None, workspace=None, stream=None):
    """The whole layer from bf16 X: Y [M][N] bf16 (one kernel at decode sizes)."""
    M, K = X.shape
    N = Wq.shape[0]
    r = 0 if L1t is None else L1t.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = Workspace(X.device)
    need = tq_layer_workspace_bytes(M, N, K, r)
    ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    _check(_lib.tq_w4a4_lr_layer(_ptr(X), _ptr(L1t) if r else None, _ptr(Wq), _ptr(s_w),
                                 _ptr(L2t) if r else None, M, N, K, r, int(had_block), _ptr(Y),
                                 _ptr(ws), ws.numel(), _stream(stream)), "tq_w4a4_lr_layer")
    return Y


def _signs(signs, K):
    """(pointer, n): a mask [K/32] (one transform) or masks [n][K/32] (n
    composed transforms, the first applied first), int32 words."""
    if signs.dim() == 2:
        _need(signs, torch.int32, (signs.shape[0], K // 32), "signs")
        return _ptr(signs), int(signs.shape[0])
    _need(signs, torch.int32, (K // 32,), "signs")
    return _ptr(signs), 1


def tq_pack_weight_rht(Rt: torch.Tensor, had_block: int, signs: torch.Tensor, Wq=None, s_w=None,
                       stream=None):
    """tq_pack_weight with the randomized Hadamard D H: `signs` is the bit
    mask [K/32] (int32 words; bit k % 32 of word k / 32 set where d_k = -1)."""
    N, K = Rt.shape
    _need(Rt, torch.float32, (N, K), "Rt")
    Wq = torch.empty(N, K // 2, dtype=torch.uint8, device=Rt.device) if Wq is None else Wq
    s_w = torch.empty(N, dtype=torch.float32, device=Rt.device) if s_w is None else s_w
    sp, n = _signs(signs, K)
    _check(_lib.tq_pack_weight_rhtn(_ptr(Rt), N, K, int(had_block), sp, n, _ptr(Wq),
                                    _ptr(s_w), _stream(stream)), "tq_pack_weight_rhtn")
    return Wq, s_w


def tq_quantize_act_rht(X: torch.Tensor, had_block: int, signs: torch.Tensor, L1t=None,
                        stream=None):
    """tq_quantize_act with the randomized Hadamard: codes of X D H (signs
    [K/32]), or of X D_1 H ... D_n H (signs [n][K/32], composed)."""
    M, K = X.shape
    _need(X, torch.bfloat16, (M, K), "X")
    r = 0 if L1t is None else L1t.shape[0]
    dev = X.device
    Xq = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
    s_x = torch.empty(M, dtype=torch.float32, device=dev)
    XL1 = torch.empty(M, r, dtype=torch.float32, device=dev) if r else None
    sp, n = _signs(signs, K)
    _check(_lib.tq_quantize_act_rhtn(_ptr(X), M, K, int(had_block), sp, n,
                                     _ptr(L1t) if r else None, r, _ptr(Xq), _ptr(s_x),
                                     _ptr(XL1) if r else None, _stream(stream)),
           "tq_quantize_act_rhtn")
    return Xq, s_x, XL1


def tq_w4a4_lr_layer_rht(X, signs, L1t, Wq, s_w, L2t, had_block, Y=None, workspace=None,
                         stream=None):
    """tq_w4a4_lr_layer with the randomized Hadamard on both sides (weights
    from tq_pack_weight_rht with the same signs)."""
    M, K = X.shape
    N = Wq.shape[0]
    r = 0 if L1t is None else L1t.shape[0]
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=X.device) if Y is None else Y
    if workspace is None:
        workspace = Workspace(X.device)
    ws = workspace.get(tq_layer_workspace_bytes(M, N, K, r)) if isinstance(workspace, Workspace) \
        else workspace
    sp, n = _signs(signs, K)
    _check(_lib.tq_w4a4_lr_layer_rhtn(_ptr(X), sp, n, _ptr(L1t) if r else None,
                                      _ptr(Wq), _ptr(s_w), _ptr(L2t) if r else None, M, N, K, r,
                                      int(had_block), _ptr(Y), _ptr(ws), ws.numel(),
                                      _stream(stream)), "tq_w4a4_lr_layer_rhtn")
    return Y


def tq_pack_gate_up(Wq_g, s_w_g, L1t_g, L2t_g, Wq_u, s_w_u, L1t_u, L2t_u, stream=None):
    """Gate and up projections (each packed by tq_pack_weight, rank r) as one
    layer of 2N interleaved channels: returns (Wq2, s_w2, L1t2, L2t2)."""
    N, Kh = Wq_g.shape
    K = 2 * Kh
    r = 0 if L1t_g is None else L1t_g.shape[0]
    dev = Wq_g.device
    Wq2 = torch.empty(2 * N, Kh, dtype=torch.uint8, device=dev)
    s_w2 = torch.empty(2 * N, dtype=torch.float32, device=dev)
    L1t2 = torch.empty(2 * r, K, dtype=torch.bfloat16, device=dev) if r else None
    L2t2 = torch.empty(2 * N, 2 * r, dtype=torch.bfloat16, device=dev) if r else None
    opt = lambda t: _ptr(t) if t is not None else None  # noqa: E731
    _check(_lib.tq_pack_gate_up(_ptr(Wq_g), _ptr(s_w_g), opt(L1t_g), opt(L2t_g), _ptr(Wq_u),
                                _ptr(s_w_u), opt(L1t_u), opt(L2t_u), N, K, r, _ptr(Wq2),
                                _ptr(s_w2), opt(L1t2), opt(L2t2), _stream(stream)),
           "tq_pack_gate_up")
    return Wq2, s_w2, L1t2, L2t2


def tq_gate_up_workspace_bytes(M: int, N: int, K: int, r2: int) -> int:
    return int(_lib.tq_gate_up_workspace_bytes(M, N, K, r2))


def tq_w4a4_lr_gate_up(X, L1t2, Wq2, s_w2, L2t2, had_block, Y=None, workspace=None, stream=None):
    """silu(gate) * up from one pass over X: Y [M][N] bf16, N = Wq2 rows / 2."""
    M, K = X.shape
    N = Wq2.shape[0] // 2
    r2 = 0 if L1t2 is None else L1t2.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = Workspace(X.device)
    need = tq_gate_up_workspace_bytes(M, N, K, r2)
    ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    _check(_lib.tq_w4a4_lr_gate_up(_ptr(X), _ptr(L1t2) if r2 else None, _ptr(Wq2), _ptr(s_w2),
                                   _ptr(L2t2) if r2 else None, M, N, K, r2, int(had_block),
                                   _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)),
           "tq_w4a4_lr_gate_up")
    return Y


def layer_forward(X, L1t, L2t, Wq, s_w, had_block, workspace=None, stream=None, out=None):
    """One layer through the two-call path: tq_quantize_act then tq_w4a4_lr_gemm."""
    Xq, s_x, XL1 = tq_quantize_act(X, had_block, L1t, stream=stream)
    return tq_w4a4_lr_gemm(Xq, s_x, Wq, s_w, XL1, L2t, Y=out, workspace=workspace,
                           stream=stream)
