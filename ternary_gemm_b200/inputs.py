"""Seeded synthetic inputs for the H-BitLinear forward.

This module holds random-number generation only -- none of the method's
arithmetic -- so that the CUDA path and the CPU oracle see identical bytes.
It imports neither of them.

The activations stand in for the inputs of the Wo / Wdown projections that
the BitNet v2 pages plot (Figures 1-3 of "BitNet v2: Native 4-bit Activations
with Hadamard Transformation for 1-bit LLMs"): a few outlier channels and most
of the mass near zero.  Weights are Gaussian latent weights that the library
ternarises.  No dataset is involved.

Rows are generated in blocks of ``BLOCK_ROWS`` from a per-block seed, so any
block can be regenerated on its own (the oracle checks sampled rows of large
configurations without materialising the whole matrix twice).

Arrays: float32 for fp32 data, uint16 for bf16 bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

BLOCK_ROWS = 1024


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even (data conversion)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One synthetic H-BitLinear problem: x [M][K] and W [N][K]."""
    name: str
    M: int
    K: int
    N: int
    dtype: str                 # "f32" or "bf16" for x and W
    x_dist: str                # "normal", "laplace", "swiglu", "swiglu_sparse"
    x_scale: float             # std (normal) / b (laplace); unused for swiglu
    outlier_frac: float        # fraction of channels that are outliers
    outlier_count: int         # explicit count (overrides frac if > 0)
    outlier_gain: float
    w_std: float
    x_seed: int
    w_seed: int
    bits: Sequence[int] = field(default=(4,))
    near_zero_frac: float = 0.0  # swiglu_sparse: share of non-outlier values replaced by U(-0.01, 0.01)

    @property
    def n_outliers(self) -> int:
        if self.outlier_count > 0:
            return self.outlier_count
        return int(round(self.outlier_frac * self.K))

    def with_rows(self, M: int) -> "Workload":
        return Workload(self.name, M, self.K, self.N, self.dtype, self.x_dist, self.x_scale,
                        self.outlier_frac, self.outlier_count, self.outlier_gain, self.w_std,
                        self.x_seed, self.w_seed, tuple(self.bits), self.near_zero_frac)

    def with_shape(self, M: int, K: int, N: int) -> "Workload":
        return Workload(self.name, M, K, N, self.dtype, self.x_dist, self.x_scale,
                        self.outlier_frac, self.outlier_count, self.outlier_gain, self.w_std,
                        self.x_seed, self.w_seed, tuple(self.bits), self.near_zero_frac)


# The five workloads: a tiny fp32 case, 1.3B-like Wo, 3B-like Wdown, 7B-like
# Wdown and the size sweeps.
WORKLOADS = {
    "tiny": Workload("tiny", 8, 256, 256, "f32", "normal", 1.0, 0.0, 4, 20.0, 0.02, 0, 1000, (4,)),
    "wo_1p3b": Workload("wo_1p3b", 4096, 2048, 2048, "bf16", "laplace", 0.1, 0.01, 0, 30.0, 0.02,
                        1, 1001, (4, 8)),
    "wdown_3b": Workload("wdown_3b", 8192, 8192, 2560, "bf16", "swiglu", 1.0, 0.005, 0, 50.0, 0.02,
                         2, 1002, (4,)),
    "wdown_7b": Workload("wdown_7b", 8192, 16384, 4096, "bf16", "swiglu_sparse", 1.0, 0.005, 0, 50.0,
                         0.015, 3, 1003, (4, 8), near_zero_frac=0.6),
    # size sweeps: the fused LN+FHT+quant kernel alone at M=65536 for each K, and
    # the whole forward at K=N=4096 for several token counts
    "sweep": Workload("sweep", 65536, 4096, 4096, "bf16", "normal", 1.0, 0.01, 0, 30.0, 0.02,
                      4, 1004, (4,)),
}
SWEEP_K1_KS = (1024, 2048, 4096, 8192, 16384, 32768)
SWEEP_FWD_MS = (1, 16, 128, 1024, 16384)


def outlier_channels(wl: Workload) -> np.ndarray:
    """Seeded choice of the outlier channels (a partial shuffle of 0..K-1)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.x_seed, 0x0C11])))
    return np.sort(rng.choice(wl.K, size=wl.n_outliers, replace=False)).astype(np.int64)


def _x_block(wl: Workload, b: int, chans: np.ndarray) -> np.ndarray:
    rows = min(BLOCK_ROWS, wl.M - b * BLOCK_ROWS)
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.x_seed, 0xB10C, b])))
    K = wl.K
    if wl.x_dist == "normal":
        x = rng.standard_normal((rows, K), dtype=np.float32) * np.float32(wl.x_scale)
    elif wl.x_dist == "laplace":
        # inverse CDF of Laplace(0, b) from uniforms in (-1/2, 1/2)
        u = rng.random((rows, K), dtype=np.float32) - np.float32(0.5)
        u = np.clip(u, np.float32(-0.4999999), np.float32(0.4999999))
        x = (-np.float32(wl.x_scale) * np.sign(u) * np.log1p(-2.0 * np.abs(u))).astype(np.float32)
    elif wl.x_dist in ("swiglu", "swiglu_sparse"):
        a = rng.standard_normal((rows, K), dtype=np.float32)
        g = rng.standard_normal((rows, K), dtype=np.float32)
        x = (a / (np.float32(1.0) + np.exp(-a)) * g).astype(np.float32)
        if wl.x_dist == "swiglu_sparse":
            mask = rng.random((rows, K), dtype=np.float32) < np.float32(wl.near_zero_frac)
            mask[:, chans] = False
            small = (rng.random((rows, K), dtype=np.float32) * np.float32(0.02) - np.float32(0.01))
            x = np.where(mask, small, x).astype(np.float32)
    else:
        raise ValueError(wl.x_dist)
    if chans.size:
        x[:, chans] *= np.float32(wl.outlier_gain)
    return x


def make_x(wl: Workload, blocks: Optional[Sequence[int]] = None) -> np.ndarray:
    """Activations [M][K] (or only the listed row blocks, concatenated).

    float32 for fp32 workloads, bf16 bits (uint16) otherwise.
    """
    chans = outlier_channels(wl)
    nb = (wl.M + BLOCK_ROWS - 1) // BLOCK_ROWS
    ids = range(nb) if blocks is None else blocks
    parts = []
    for b in ids:
        xb = _x_block(wl, b, chans)
        parts.append(xb if wl.dtype == "f32" else f32_to_bf16_bits(xb))
    return np.concatenate(parts, axis=0) if len(parts) > 1 else parts[0]


def make_x_rows(wl: Workload, rows: Sequence[int]) -> np.ndarray:
    """Selected rows of make_x(wl), regenerating only their blocks."""
    rows = np.asarray(rows, dtype=np.int64)
    blocks = sorted(set(int(r) // BLOCK_ROWS for r in rows))
    data = {b: make_x(wl, [b]) for b in blocks}
    return np.stack([data[int(r) // BLOCK_ROWS][int(r) % BLOCK_ROWS] for r in rows], axis=0)


def make_w(wl: Workload) -> np.ndarray:
    """Latent weights [N][K] ~ N(0, w_std^2) (float32 or bf16 bits)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([wl.w_seed, 0x3E16])))
    w = rng.standard_normal((wl.N, wl.K), dtype=np.float32) * np.float32(wl.w_std)
    return w if wl.dtype == "f32" else f32_to_bf16_bits(w)


def sample_rows(M: int, n: int, seed: int = 7) -> np.ndarray:
    """First, last and n seeded distinct rows in between (sorted, unique)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    inner = rng.choice(M, size=min(n, M), replace=False) if M > 0 else np.zeros(0, np.int64)
    return np.unique(np.concatenate([[0, M - 1], inner]).astype(np.int64))
