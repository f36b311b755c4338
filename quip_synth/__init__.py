"""Seeded synthetic workloads for one linear layer (inputs only).

This module is shared by the FP64 oracle (tests, bench baseline) and the CUDA
path.  It draws weights ``W`` and calibration activations ``X`` and nothing
else: it holds none of the quantizer's arithmetic (no Hessian, no transform, no
factorisation, no rounding).  The random orthogonal transforms are *not* drawn
here: each side derives them from the integer ``seed`` with its own
implementation of the counter-based SplitMix64 generator.

The shapes stand in for the QuIP paper's setting (Experiments, "Setup.":
OPT / Llama-2 linear layers, 128 random 2048-token C4 segments as calibration
data); neither the weights nor C4 are available, so both are synthetic:

* ``W`` — i.i.d. N(0, sigma^2); a fraction ``w_outlier_frac`` of the flat
  indices (drawn without replacement) is multiplied by ``w_outlier_mult``;
  then rounded to bfloat16 (round-to-nearest-even) unless ``dtype='f32'``.
* ``X`` — i.i.d. N(0, 1) tokens x channels; either a fraction
  ``x_outlier_frac`` of channels (drawn without replacement) scaled by
  ``x_outlier_mult``, or per-channel log-normal(0, 1) multipliers; then
  rounded to bfloat16 unless ``dtype='f32'``.

Draw order from ``numpy.random.Generator(PCG64(seed))``: W, W-outlier indices,
X, X channel scales.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Tuple

import numpy as np

__all__ = ["Side", "LayerConfig", "CONFIGS", "make_layer", "to_bf16_bits",
           "bf16_bits_to_f32", "round_to_bf16", "calibration_chunks"]


@dataclass(frozen=True)
class Side:
    """Incoherence transform requested for one side of W.

    kind: 'hadamard' (dimension a power of two), 'kronecker' (p*q == dim) or
    'identity'; permute: a random permutation of the coordinates is applied
    before the structured transform.
    """
    kind: str
    p: int = 0
    q: int = 0
    permute: bool = False


@dataclass(frozen=True)
class LayerConfig:
    name: str
    m: int                      # output rows of W
    n: int                      # input columns of W (= Hessian order)
    N: int                      # calibration tokens
    m_side: Side
    n_side: Side
    block: int                  # LDLQ column block
    bits: int
    sigma: float = 0.02
    w_outlier_frac: float = 0.0
    w_outlier_mult: float = 10.0
    x_outlier_frac: float = 0.0
    x_outlier_mult: float = 20.0
    x_lognormal: bool = False
    dtype: str = "bf16"         # storage type of W and X: 'bf16' or 'f32'
    damp: float = 0.01
    seed: int = 0

    @property
    def weights(self) -> int:
        return self.m * self.n


CONFIGS: Dict[str, LayerConfig] = {
    # tiny layer: fp32 storage, log-normal channel scales, Hadamard on both
    # sides (64 and 128), block 32, 2-bit.
    "tiny": LayerConfig("tiny", 64, 128, 1024, Side("hadamard"), Side("hadamard"),
                        block=32, bits=2, dtype="f32", x_lognormal=True),
    # Llama-2-7B-shaped attention projection.
    "attn7b": LayerConfig("attn7b", 4096, 4096, 8192, Side("hadamard"), Side("hadamard"),
                          block=128, bits=2, w_outlier_frac=0.001, x_outlier_frac=0.01),
    # Llama-2-7B MLP up projection: Kronecker 86x128 on the 11008 output side.
    "up7b": LayerConfig("up7b", 11008, 4096, 16384, Side("kronecker", 86, 128), Side("hadamard"),
                        block=128, bits=3, w_outlier_frac=0.001, x_outlier_frac=0.01),
    # Llama-2-7B MLP down projection: Kronecker 86x128 on the 11008 input side.
    "down7b": LayerConfig("down7b", 4096, 11008, 16384, Side("hadamard"), Side("kronecker", 86, 128),
                          block=128, bits=4, w_outlier_frac=0.001, x_outlier_frac=0.01),
    # Llama-2-70B-shaped MLP gate: Kronecker 224x128 on the 28672 output side.
    "gate70b": LayerConfig("gate70b", 28672, 8192, 32768, Side("kronecker", 224, 128), Side("hadamard"),
                           block=128, bits=2, sigma=0.015, w_outlier_frac=0.001, x_outlier_frac=0.01),
}


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), returned as float32."""
    return bf16_bits_to_f32(to_bf16_bits(a))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round-to-nearest-even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_layer(cfg: LayerConfig, rows: Tuple[int, int] | None = None) -> Dict[str, np.ndarray]:
    """Draw (W, X) for ``cfg``.

    Returns a dict with float32 arrays ``W`` (m x n) and ``X`` (N x n) holding
    exactly the stored values (bf16-representable unless dtype is 'f32'), and,
    for bf16 configs, the raw bf16 bit patterns ``W_bf16`` / ``X_bf16``.
    """
    rng = np.random.Generator(np.random.PCG64(cfg.seed))
    m, n, N = cfg.m, cfg.n, cfg.N
    W = rng.standard_normal((m, n), dtype=np.float64) * cfg.sigma
    if cfg.w_outlier_frac > 0:
        k = int(round(cfg.w_outlier_frac * m * n))
        idx = rng.choice(m * n, size=k, replace=False)
        W.reshape(-1)[idx] *= cfg.w_outlier_mult
    W = W.astype(np.float32)
    X = rng.standard_normal((N, n), dtype=np.float32)
    if cfg.x_lognormal:
        scale = np.exp(rng.standard_normal(n)).astype(np.float32)
        X *= scale[None, :]
    elif cfg.x_outlier_frac > 0:
        k = int(round(cfg.x_outlier_frac * n))
        ch = rng.choice(n, size=k, replace=False)
        X[:, ch] *= np.float32(cfg.x_outlier_mult)
    out: Dict[str, np.ndarray] = {}
    if cfg.dtype == "bf16":
        wb = to_bf16_bits(W)
        xb = to_bf16_bits(X)
        out["W_bf16"], out["X_bf16"] = wb, xb
        W, X = bf16_bits_to_f32(wb), bf16_bits_to_f32(xb)
    out["W"], out["X"] = W, X
    return out


def random_layer(m: int, n: int, N: int, seed: int, dtype: str = "f32", sigma: float = 0.02,
                 x_outlier_frac: float = 0.0, lognormal: bool = True) -> Dict[str, np.ndarray]:
    """Small ad-hoc layer (ragged sizes for edge-case tests), same recipe."""
    cfg = LayerConfig("adhoc", m, n, N, Side("identity"), Side("identity"), block=n, bits=2,
                      sigma=sigma, x_outlier_frac=x_outlier_frac, x_lognormal=lognormal,
                      dtype=dtype, seed=seed)
    return make_layer(cfg)


def calibration_chunks(n: int, N: int, chunk: int, seed: int, x_outlier_frac: float = 0.01,
                       x_outlier_mult: float = 20.0):
    """Calibration activations streamed in token chunks, the recipe of the
    Llama-shaped workloads (i.i.d. N(0, 1), a fraction of channels scaled by
    ``x_outlier_mult``, rounded to bf16) at a token count too large to hold
    at once: the QuIP paper calibrates on 128 segments of 2048 tokens
    (Experiments, "Setup.").  The outlier channels are drawn once from
    PCG64(seed); chunk c from PCG64(seed + 1 + c).  Yields (first token,
    float32 values, bf16 bit patterns) per chunk of at most ``chunk`` tokens."""
    rng = np.random.Generator(np.random.PCG64(seed))
    k = int(round(x_outlier_frac * n))
    ch = rng.choice(n, size=k, replace=False) if k > 0 else np.zeros(0, dtype=np.int64)
    for c, a in enumerate(range(0, N, chunk)):
        b = min(N, a + chunk)
        r = np.random.Generator(np.random.PCG64(seed + 1 + c))
        X = r.standard_normal((b - a, n), dtype=np.float32)
        X[:, ch] *= np.float32(x_outlier_mult)
        xb = to_bf16_bits(X)
        yield a, bf16_bits_to_f32(xb), xb
