"""Seeded synthetic layer inputs (activations, low-rank factors, residual).

Recipe (one reading of the pages per point):

* X is bf16 with N(0,1) elements; a seeded choice of input channels is scaled
  (x20 on 2 of 256 channels for the tiny layer, x30 on round(0.01*K) channels
  otherwise) before the bf16 rounding.  This mimics the activation outliers
  that motivate rotation in CoQuant (section 3, "uniform quantization is
  sensitive to outliers").
* W = U diag(sigma) V^T with U [K x p], V [N x p] the sign-fixed thin
  Householder QR factors of seeded Gaussians, p = min(K, N), and a slowly
  decaying spectrum sigma_i ~ i^-1/2 (TwinQuant notes, Figure 1: slow spectral
  decay of LLM weights).  The tiny layer uses sigma_i = 0.02*sqrt(256)*i^-1/2
  literally; the others are scaled so that W has elementwise std 0.02.
* L1 = U_r sqrt(Sigma_r), L2 = sqrt(Sigma_r) V_r^T, both rounded to bf16, and
  the residual R = W - bf16(L1) bf16(L2) is formed in fp64 and stored fp32, so
  the two branches complement each other exactly (SVDQuant-style split quoted
  in the TwinQuant notes, section 02.A).

Storage follows nn.Linear ([out][in]): X [M][K], L1t = L1^T [r][K],
L2t = L2^T [N][r], Rt = R^T [N][K].

Seeds: X uses `seed`, U `seed+1`, V `seed+2`, the outlier permutation
`seed+3`.  Random numbers are always drawn on the CPU generator so they do not
depend on the device; only the QR and the products may run on a GPU for the
large shapes, which changes the bytes at the rounding level but not their
distribution.  Both the oracle and the CUDA path always consume the same bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class LayerShape:
    name: str
    M: int
    K: int
    N: int
    r: int
    had_block: int = 128
    outlier_channels: int | None = None  # None -> round(0.01*K)
    outlier_scale: float = 30.0
    sigma_literal: bool = False          # tiny layer: sigma_i = 0.02*sqrt(256)*i^-1/2
    weight_std: float = 0.02

    def with_(self, **kw) -> "LayerShape":
        return replace(self, **kw)

    @property
    def n_outliers(self) -> int:
        if self.outlier_channels is not None:
            return self.outlier_channels
        return int(round(0.01 * self.K))


# The layer shapes of the workloads (Llama-3 projections).  M lists are the
# token counts each shape is exercised at.
CONFIGS: dict[str, LayerShape] = {
    "tiny": LayerShape("tiny", M=16, K=256, N=256, r=16, had_block=256,
                       outlier_channels=2, outlier_scale=20.0, sigma_literal=True),
    "decode": LayerShape("decode", M=16, K=4096, N=4096, r=32),
    "prefill_gateup": LayerShape("prefill_gateup", M=2048, K=4096, N=14336, r=64),
    "prefill_down": LayerShape("prefill_down", M=2048, K=14336, N=4096, r=64),
    "large_gateup": LayerShape("large_gateup", M=4096, K=8192, N=28672, r=128),
    "large_down": LayerShape("large_down", M=4096, K=28672, N=8192, r=128),
    "sweep": LayerShape("sweep", M=4096, K=4096, N=4096, r=64),
}
DECODE_M = (1, 16, 128)
SWEEP_RANKS = (0, 32, 64, 128, 256, 512)
SWEEP_M = (1, 4, 16, 64, 256, 1024, 4096, 8192)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def make_activations(shape: LayerShape, seed: int = 0, M: int | None = None) -> torch.Tensor:
    """X [M][K] bf16 (CPU) with seeded outlier channels."""
    M = shape.M if M is None else M
    K = shape.K
    x = torch.randn(M, K, generator=_gen(seed), dtype=torch.float32)
    n_out = shape.n_outliers
    if n_out > 0:
        perm = torch.randperm(K, generator=_gen(seed + 3))
        ch = perm[:n_out]
        x[:, ch] *= shape.outlier_scale
    return x.to(torch.bfloat16)


def _orthonormal(rows: int, cols: int, seed: int, device: str) -> torch.Tensor:
    """Sign-fixed thin QR factor of a seeded Gaussian (Haar-distributed columns)."""
    a = torch.randn(rows, cols, generator=_gen(seed), dtype=torch.float64)
    a = a.to(device)
    q, rr = torch.linalg.qr(a, mode="reduced")
    d = torch.sign(torch.diagonal(rr))
    d[d == 0] = 1.0
    return q * d.unsqueeze(0)


def _spectrum(shape: LayerShape, p: int, device: str) -> torch.Tensor:
    i = torch.arange(1, p + 1, dtype=torch.float64, device=device)
    if shape.sigma_literal:
        return 0.02 * math.sqrt(256.0) * i.pow(-0.5)
    sig = i.pow(-0.5)
    # ||W||_F^2 = sum sigma_i^2 for orthonormal U, V; scale to std weight_std.
    target = shape.weight_std ** 2 * shape.K * shape.N
    return sig * math.sqrt(target / float((sig * sig).sum()))


def make_weights(shape: LayerShape, seed: int = 0, device: str = "cpu") -> dict:
    """Low-rank factors and residual of W = U diag(sigma) V^T.

    Returns CPU tensors: L1t bf16 [r][K], L2t bf16 [N][r], Rt fp32 [N][K].
    """
    K, N, r = shape.K, shape.N, shape.r
    p = min(K, N)
    if r > p:
        raise ValueError(f"rank {r} exceeds min(K, N) = {p}")
    U = _orthonormal(K, p, seed + 1, device)
    V = _orthonormal(N, p, seed + 2, device)
    sig = _spectrum(shape, p, device)
    W = (U * sig.unsqueeze(0)) @ V.T                      # [K][N] fp64
    if r > 0:
        sq = sig[:r].sqrt()
        L1 = (U[:, :r] * sq.unsqueeze(0)).to(torch.bfloat16)       # [K][r]
        L2 = (sq.unsqueeze(1) * V[:, :r].T).to(torch.bfloat16)     # [r][N]
        R = W - L1.double() @ L2.double()
        L1t = L1.T.contiguous().cpu()
        L2t = L2.T.contiguous().cpu()
    else:
        R = W
        L1t = torch.empty(0, K, dtype=torch.bfloat16)
        L2t = torch.empty(N, 0, dtype=torch.bfloat16)
    Rt = R.T.contiguous().to(torch.float32).cpu()
    del U, V, W, R
    return {"L1t": L1t, "L2t": L2t, "Rt": Rt}


def make_layer(shape: LayerShape, seed: int = 0, M: int | None = None,
               device: str = "cpu") -> dict:
    """All inputs of one layer: X, L1t, L2t, Rt (CPU tensors) plus the shape."""
    out = make_weights(shape, seed=seed, device=device)
    out["X"] = make_activations(shape, seed=seed, M=M)
    out["shape"] = shape if M is None else shape.with_(M=M)
    return out
