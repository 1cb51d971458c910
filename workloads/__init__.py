"""Seeded synthetic inputs and workload shapes for the NVFP4 GEMM + epilogue path.

This module is shared by the CUDA path (tests, bench) and by the CPU oracle. It holds
only shapes and random-number draws: no quantisation, GEMM, normalisation or
activation arithmetic lives here.

Distributions follow the workloads of the DiT layer described in "Serving sub-second
Ideogram v4 without quality loss" (fal), sections "Running the transformer in FP4"
and "Epilogue fusion in brief": activations N(0, 1) with a few outlier input
channels scaled x20, weights N(0, std 1/sqrt(K)), RMSNorm weights 1 + N(0, 0.1).
Every tensor is drawn from its own numpy substream ``default_rng([seed, stream])``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

# Substream ids, one per drawn tensor.
_S_ACT, _S_WEIGHT, _S_NORM_W, _S_OUTLIER, _S_NORM_W2 = 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class Workload:
    """One GEMM + epilogue problem: A (M x K) @ B (N x K)^T, then ``op``.

    op: "plain" | "rmsnorm" | "swiglu".
    For "swiglu", N is the width of the gate|up weight (2 * Nh) and the output is M x Nh.
    For "rmsnorm", the first ``n_norm_cols`` output columns are normalised per head of
    ``head_dim`` columns; the rest pass through.
    """

    name: str
    M: int
    K: int
    N: int
    op: str
    head_dim: int = 0
    n_norm_cols: int = 0
    eps: float = 1e-6
    outliers: int = 0            # number of activation input channels scaled x20
    requant: bool = False        # swiglu output re-quantised to NVFP4
    weight_std: Optional[float] = None  # default 1/sqrt(K)
    seed: int = 0

    @property
    def n_out(self) -> int:
        return self.N // 2 if self.op == "swiglu" else self.N

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    def std(self) -> float:
        return self.weight_std if self.weight_std is not None else 1.0 / np.sqrt(self.K)


def outlier_count(K: int, frac: float = 1e-3) -> int:
    """0.1 % of the input channels, rounded to nearest, at least one."""
    return max(1, int(round(frac * K)))


# Named workloads: the tiny QK-norm case, the SwiGLU case, the 1K-image QKV and FFN
# blocks (M = 64 x 64 latent patches = 4096 tokens) and the batched sweep over M.
def qk_norm_tiny() -> Workload:
    return Workload("qknorm_tiny_256x1024x1024_hd256", 256, 1024, 1024, "rmsnorm",
                    head_dim=256, n_norm_cols=1024, outliers=8, weight_std=1.0 / 32)


def swiglu_1024() -> Workload:
    return Workload("swiglu_1024x3072x16384", 1024, 3072, 2 * 8192, "swiglu",
                    outliers=outlier_count(3072))


def qkv(M: int = 4096, head_dim: int = 256) -> Workload:
    # 12 heads x 256 (or 24 x 128) for each of Q, K, V: N = 9216; Q and K normalised.
    return Workload(f"qkv_{M}x3072x9216_hd{head_dim}", M, 3072, 9216, "rmsnorm",
                    head_dim=head_dim, n_norm_cols=6144, outliers=outlier_count(3072))


def ffn_up(M: int = 4096, requant: bool = True) -> Workload:
    return Workload(f"ffn_up_{M}x3072x24576{'_q' if requant else ''}", M, 3072, 2 * 12288,
                    "swiglu", outliers=outlier_count(3072), requant=requant)


def ffn_down(M: int = 4096) -> Workload:
    return Workload(f"ffn_down_{M}x12288x3072", M, 12288, 3072, "plain",
                    outliers=0)


SWEEP_M = (1024, 4096, 8192, 16384)


def sweep() -> list:
    out = []
    for M in SWEEP_M:
        out += [qkv(M, 128), qkv(M, 256), ffn_up(M, True)]
    return out


# ----------------------------------------------------------------------------------
# Random draws
# ----------------------------------------------------------------------------------

def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, stream])


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """float array -> CPU torch.bfloat16 tensor (the inputs' storage type)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def activations(M: int, K: int, outliers: int, seed: int = 0, stream: int = _S_ACT) -> torch.Tensor:
    """A ~ N(0, 1), with ``outliers`` input channels (columns of A) scaled by 20."""
    a = _rng(seed, stream).standard_normal((M, K), dtype=np.float32)
    if outliers:
        idx = _rng(seed, _S_OUTLIER).choice(K, size=outliers, replace=False)
        a[:, idx] *= 20.0
    return to_bf16(a)


def weights(N: int, K: int, std: float, seed: int = 0, stream: int = _S_WEIGHT) -> torch.Tensor:
    """B ~ N(0, std^2), N x K (K-major: one output column per row)."""
    return to_bf16(_rng(seed, stream).standard_normal((N, K), dtype=np.float32) * np.float32(std))


def norm_weight(head_dim: int, seed: int = 0, stream: int = _S_NORM_W) -> np.ndarray:
    """RMSNorm weight w = 1 + N(0, 0.1^2), length head_dim, float32."""
    return (1.0 + 0.1 * _rng(seed, stream).standard_normal(head_dim)).astype(np.float32)


def norm_weight_columns(wl: Workload) -> np.ndarray:
    """Per-column RMSNorm weight for the first n_norm_cols columns.

    The Q block uses w_q and the K block w_k, each of length head_dim and shared by all
    heads of its block; with n_norm_cols == N (the tiny case) a single w is tiled.
    """
    hd = wl.head_dim
    if wl.n_norm_cols == wl.N:
        return np.tile(norm_weight(hd, wl.seed), wl.N // hd)
    half = wl.n_norm_cols // 2
    wq = np.tile(norm_weight(hd, wl.seed, _S_NORM_W), half // hd)
    wk = np.tile(norm_weight(hd, wl.seed, _S_NORM_W2), half // hd)
    return np.concatenate([wq, wk]).astype(np.float32)


def make_inputs(wl: Workload) -> dict:
    """All seeded inputs of a workload as CPU tensors / arrays."""
    d = {"a": activations(wl.M, wl.K, wl.outliers, wl.seed),
         "b": weights(wl.N, wl.K, wl.std(), wl.seed)}
    if wl.op == "rmsnorm":
        d["w"] = norm_weight_columns(wl)
    return d


def fp4_codes_exact(rows: int, cols: int, seed: int, stream: int) -> np.ndarray:
    """Random E2M1 codes 0..15 (uint8, one per element) for exact-arithmetic cases."""
    return _rng(seed, stream).integers(0, 16, size=(rows, cols), dtype=np.uint8)


def pow2_scales_exact(rows: int, nblk: int, seed: int, stream: int,
                      lo: int = -2, hi: int = 0) -> np.ndarray:
    """Random power-of-two block scales 2^lo..2^hi as float64, rows x nblk."""
    e = _rng(seed, stream).integers(lo, hi + 1, size=(rows, nblk))
    return np.ldexp(1.0, e)
