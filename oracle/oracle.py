"""ctypes wrapper of the fp64 C oracle (test infrastructure only)."""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build_oracle import build as _build

_lib = None
_P = ctypes.c_void_p
_L = ctypes.c_long


def _load():
    global _lib
    if _lib is None:
        path = _build()
        lib = ctypes.CDLL(path)
        lib.orc_hadamard_entry.restype = ctypes.c_double
        lib.orc_hadamard_entry.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.orc_rotate.argtypes = [_P, _L, _L, ctypes.c_int, _P]
        lib.orc_quantize_sym.argtypes = [_P, _L, _L, ctypes.c_int, _P, _P, _P]
        lib.orc_quantize_asym.argtypes = [_P, _L, _L, ctypes.c_int, _P, _P, _P, _P]
        lib.orc_pack_int4.argtypes = [_P, _L, _L, _P]
        lib.orc_unpack_int4.argtypes = [_P, _L, _L, _P]
        lib.orc_int_gemm.restype = ctypes.c_long
        lib.orc_int_gemm.argtypes = [_P, _P, _L, _L, _L, _P]
        lib.orc_round_bf16.restype = ctypes.c_double
        lib.orc_round_bf16.argtypes = [ctypes.c_double]
        lib.orc_lowrank.argtypes = [_P, _P, _P, _L, _L, _L, _L, ctypes.c_int, _P, _P]
        lib.orc_epilogue.argtypes = [_P, _P, _P, _P, _L, _L, _P]
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    """Exact conversion to a contiguous fp64 numpy array (torch tensors welcome)."""
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def num_threads() -> int:
    return int(_load().orc_num_threads())


def set_num_threads(n: int) -> None:
    _load().orc_set_num_threads(int(n))


def hadamard(b: int) -> np.ndarray:
    """Dense normalised Sylvester Hadamard matrix H_b (fp64)."""
    lib = _load()
    return np.array([[lib.orc_hadamard_entry(b, i, j) for j in range(b)] for i in range(b)])


def signs_from_bits(bits, K: int) -> np.ndarray:
    """The sign vector d [K] (+1 / -1, fp64) of the randomized Hadamard
    transform from its bit mask: K / 32 little-endian uint32 words, bit
    (k % 32) of word k / 32 set where d_k = -1."""
    w = np.ascontiguousarray(np.asarray(bits, dtype=np.uint32))
    if w.ndim == 2:  # n masks (composed transforms): rows of signs
        return np.stack([signs_from_bits(row, K) for row in w])
    assert w.size * 32 >= K, (w.size, K)
    neg = np.unpackbits(w.view(np.uint8), bitorder="little")[:K]
    return np.where(neg == 1, -1.0, 1.0)


def rotate(x, b: int, signs=None) -> np.ndarray:
    """Rows of x times diag(H_b, ..., H_b) (fp64); with `signs` (the +-1
    vector d), rows of x times D diag(H_b, ...): the randomized Hadamard
    transform, signs first, then the Hadamard blocks.  `signs` of shape
    (n, K) composes n randomized Hadamard transforms, the first row's
    first: x D_1 H D_2 H ... D_n H."""
    x = _f64(x)
    rows, K = x.shape
    assert K % b == 0
    if signs is None:
        masks = [None]
    else:
        d = np.asarray(signs, dtype=np.float64)
        masks = list(d) if d.ndim == 2 else [d]
    for m in masks:
        if m is not None:
            assert m.shape == (K,)
            x = np.ascontiguousarray(x * m[None, :])
        out = np.empty_like(x)
        _load().orc_rotate(_ptr(x), rows, K, int(b), _ptr(out))
        x = out
    return x


def quantize_sym(v, qmax: int = 7):
    """Per-row symmetric RoundClip: returns (codes int8, scales fp64, v/s fp64)."""
    v = _f64(v)
    rows, K = v.shape
    q = np.empty((rows, K), dtype=np.int8)
    s = np.empty(rows, dtype=np.float64)
    t = np.empty((rows, K), dtype=np.float64)
    _load().orc_quantize_sym(_ptr(v), rows, K, int(qmax), _ptr(q), _ptr(s), _ptr(t))
    return q, s, t


def pack_int4(q) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    rows, K = q.shape
    assert K % 32 == 0
    out = np.empty((rows, K // 2), dtype=np.uint8)
    _load().orc_pack_int4(_ptr(q), rows, K, _ptr(out))
    return out


def unpack_int4(p) -> np.ndarray:
    p = np.ascontiguousarray(p, dtype=np.uint8)
    rows, K2 = p.shape
    K = 2 * K2
    assert K % 32 == 0
    q = np.empty((rows, K), dtype=np.int8)
    _load().orc_unpack_int4(_ptr(p), rows, K, _ptr(q))
    return q


def int_gemm(qa, qb) -> np.ndarray:
    """acc = qa qb^T in int64; raises if the INT32 bound 49K is violated."""
    qa = np.ascontiguousarray(qa, dtype=np.int8)
    qb = np.ascontiguousarray(qb, dtype=np.int8)
    M, K = qa.shape
    N, K2 = qb.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int64)
    bad = _load().orc_int_gemm(_ptr(qa), _ptr(qb), M, N, K, _ptr(acc))
    if bad:
        raise ValueError(f"{bad} accumulators exceed 49*K or int32")
    return acc


def round_bf16(x) -> np.ndarray:
    lib = _load()
    x = _f64(x)
    return np.vectorize(lib.orc_round_bf16, otypes=[np.float64])(x) if x.size else x.copy()


def lowrank(X, L1t, L2t, round_mid: bool = True):
    """(XL1 [M][r], lr [M][N]) of the low-rank branch (fp64)."""
    X, L1t, L2t = _f64(X), _f64(L1t), _f64(L2t)
    M, K = X.shape
    r = L1t.shape[0]
    N = L2t.shape[0]
    XL1 = np.zeros((M, r), dtype=np.float64)
    lr = np.zeros((M, N), dtype=np.float64)
    if r > 0:
        assert L1t.shape == (r, K) and L2t.shape == (N, r)
        _load().orc_lowrank(_ptr(X), _ptr(L1t), _ptr(L2t), M, N, K, r,
                            1 if round_mid else 0, _ptr(XL1), _ptr(lr))
    return XL1, lr


def epilogue(s_x, s_w, acc, lr=None) -> np.ndarray:
    s_x, s_w = _f64(s_x), _f64(s_w)
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    M, N = acc.shape
    Y = np.empty((M, N), dtype=np.float64)
    lrp = None
    if lr is not None:
        lr = _f64(lr)
        lrp = _ptr(lr)
    _load().orc_epilogue(_ptr(s_x), _ptr(s_w), _ptr(acc), lrp, M, N, _ptr(Y))
    return Y


def quantize_act(X, b: int, L1t=None, signs=None) -> dict:
    """Oracle of tq_quantize_act: rotation (randomized with `signs`),
    per-token codes, scales, X L1 (of the unrotated X)."""
    Xd = _f64(X)
    q, s, t = quantize_sym(rotate(Xd, b, signs))
    out = {"qx": q, "s_x": s, "t_x": t, "Xq": pack_int4(q)}
    if L1t is not None and _f64(L1t).shape[0] > 0:
        L1d = _f64(L1t)
        XL1, _ = lowrank(Xd, L1d, np.zeros((0, L1d.shape[0])))
        out["XL1"] = XL1
    return out


def pack_weight(Rt, b: int, signs=None) -> dict:
    """Oracle of tq_pack_weight: rotation of R^T rows (by D H with
    `signs`: row n of R^T D H is column n of (D H)^T R), per-channel
    codes / scales."""
    q, s, t = quantize_sym(rotate(_f64(Rt), b, signs))
    return {"qw": q, "s_w": s, "t_w": t, "Wq": pack_int4(q)}


def layer(X, L1t, L2t, Rt, b: int, round_mid: bool = True, signs=None) -> dict:
    """The whole layer: dequant(Q4(X H) Q4(H^T R)) + bf16(X L1) L2, in fp64;
    with `signs`, H is the randomized D H on both sides."""
    a = quantize_act(X, b, signs=signs)
    w = pack_weight(Rt, b, signs=signs)
    acc = int_gemm(a["qx"], w["qw"])
    XL1, lr = lowrank(X, L1t, L2t, round_mid=round_mid)
    Y64 = epilogue(a["s_x"], w["s_w"], acc, lr if _f64(L1t).shape[0] > 0 else None)
    out = dict(a)
    out.update(w)
    out.update({"acc": acc, "XL1": XL1, "lr": lr, "Y64": Y64, "Ybf16": round_bf16(Y64)})
    return out


def swiglu(g, u) -> np.ndarray:
    """silu(g) * u = g / (1 + exp(-g)) * u, elementwise in fp64: the gate /
    up pair's output from the two layers' fp64 outputs."""
    g, u = _f64(g), _f64(u)
    return g / (1.0 + np.exp(-g)) * u


def quantize_asym(v, qmax: int = 15):
    """Per-row asymmetric RoundClip (CoQuant Eq. (1), zero-point = row min):
    returns (codes uint8 in [0, qmax], scales, zero-points, (v - z)/s), fp64."""
    v = _f64(v)
    rows, K = v.shape
    q = np.empty((rows, K), dtype=np.uint8)
    s = np.empty(rows, dtype=np.float64)
    z = np.empty(rows, dtype=np.float64)
    t = np.empty((rows, K), dtype=np.float64)
    _load().orc_quantize_asym(_ptr(v), rows, K, int(qmax), _ptr(q), _ptr(s), _ptr(z), _ptr(t))
    return q, s, z, t


def layer_asym(X, L1t, L2t, Rt, b: int) -> dict:
    """The layer with per-token asymmetric activations: the rotated X
    quantized as Q(x) = s_x q + z_x (q in [0, 15]), the weights as in layer():
    Y = s_x s_w (q . qw) + z_x s_w (sum_k qw) + bf16(X L1) L2, in fp64."""
    q, s_x, z_x, t = quantize_asym(rotate(_f64(X), b))
    w = pack_weight(Rt, b)
    qw = w["qw"].astype(np.int64)
    acc = q.astype(np.int64) @ qw.T                     # exact in int64
    wsum = qw.sum(axis=1)
    XL1, lr = lowrank(X, L1t, L2t)
    Y64 = (s_x[:, None] * acc + z_x[:, None] * wsum[None, :]) * w["s_w"][None, :]
    if _f64(L1t).shape[0] > 0:
        Y64 = Y64 + lr
    out = {"qa": q, "s_x": s_x, "z_x": z_x, "t_x": t, "acc": acc, "wsum": wsum,
           "XL1": XL1, "lr": lr, "Y64": Y64}
    out.update(w)
    return out


def layer_qlr(X, L1t, L2t, Rt, b: int) -> dict:
    """The layer with the INT4 low-rank branch (TwinQuant Figure 4): X L1 from
    the same rotated activation codes and INT4 codes of H^T L1 (per column),
    dequantized, requantized per token to INT4, times INT4 codes of L2 (per
    output channel); Y = s_x s_w (qx . qw) + s_xl1 s_L2 (q_xl1 . q_L2), fp64."""
    a = quantize_act(X, b)
    w = pack_weight(Rt, b)
    l1 = pack_weight(L1t, b)                 # rows of L1^T rotated like weight rows
    acc1 = int_gemm(a["qx"], l1["qw"])       # [M][r], exact
    xl1 = a["s_x"][:, None] * l1["s_w"][None, :] * acc1
    qxl1, s_xl1, t_xl1 = quantize_sym(xl1)
    ql2, s_l2, t_l2 = quantize_sym(_f64(L2t))  # per output channel over r, no rotation
    acc = int_gemm(a["qx"], w["qw"])
    acc2 = int_gemm(qxl1, ql2)
    Y64 = (a["s_x"][:, None] * w["s_w"][None, :] * acc
           + s_xl1[:, None] * s_l2[None, :] * acc2)
    out = dict(a)
    out.update(w)
    out.update({"qL1": l1["qw"], "s_L1": l1["s_w"], "acc1": acc1, "xl1": xl1, "qxl1": qxl1,
                "s_xl1": s_xl1, "t_xl1": t_xl1, "qL2": ql2, "s_L2": s_l2, "t_L2": t_l2,
                "acc": acc, "acc2": acc2, "Y64": Y64})
    return out
