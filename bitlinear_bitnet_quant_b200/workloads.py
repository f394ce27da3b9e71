"""Seeded synthetic inputs shaped like the BitNet workloads.

This module holds no arithmetic of the BitLinear method: it only draws
random numbers and stores them in the input dtypes (fp32, or bf16 kept as
raw uint16 bit patterns).  Both the CUDA path and the CPU oracle receive the
very same arrays from here, so a parity test never depends on two random
generators agreeing.

Recipes (the shapes and distributions the BitNet pages' workloads imply):

* weights: fp32 ~ N(0, 0.02); the ternary codes come from absmean
  quantisation downstream (about 31 % zeros for Gaussian weights);
* activations: N(0, 1) with a fraction of "entry" outliers (distinct random
  positions scaled by a factor) or "channel" outliers (random columns scaled
  for every token), or heavy-tailed Student-t (nu = 3) for the BitNet v2
  H-BitLinear a4 case, whose outlier channels motivate the Hadamard step.

Outlier counts are ``round(p * count)``.  Generators are numpy PCG64 streams:
activations use ``default_rng(seed)``, weights ``default_rng(seed + 1000)``.
"""
from __future__ import annotations

import numpy as np

WEIGHT_SEED_OFFSET = 1000


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) and return the uint16 bits.

    Inputs must be finite.  This is only the storage conversion of a
    synthetic input, not a step of the method.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def gaussian(rng: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    return (rng.standard_normal(size=shape) * sigma).astype(np.float32)


def student_t(rng: np.random.Generator, shape, nu: int = 3) -> np.ndarray:
    """z / sqrt(chi2_nu / nu), chi2_nu drawn as a sum of nu squared normals."""
    z = rng.standard_normal(size=shape)
    chi2 = np.zeros(shape, dtype=np.float64)
    for _ in range(nu):
        chi2 += rng.standard_normal(size=shape) ** 2
    return (z / np.sqrt(chi2 / nu)).astype(np.float32)


def add_entry_outliers(rng, x: np.ndarray, frac: float, factor: float) -> np.ndarray:
    """Scale round(frac * x.size) distinct random entries by ``factor``."""
    x = x.copy()
    n = int(round(frac * x.size))
    if n:
        idx = rng.choice(x.size, size=n, replace=False)
        flat = x.reshape(-1)
        flat[idx] *= np.float32(factor)
    return x


def add_channel_outliers(rng, x: np.ndarray, frac: float, factor: float) -> np.ndarray:
    """Scale round(frac * K) random columns (all tokens) by ``factor``."""
    x = x.copy()
    K = x.shape[-1]
    n = int(round(frac * K))
    if n:
        cols = rng.choice(K, size=n, replace=False)
        x[..., cols] *= np.float32(factor)
    return x


def weights(N: int, K: int, seed: int = 0, sigma: float = 0.02) -> np.ndarray:
    rng = np.random.default_rng(seed + WEIGHT_SEED_OFFSET)
    return gaussian(rng, (N, K), sigma)


# ----------------------------------------------------------------------------
# Named workloads.  Each returns a dict with the activation input ("x", fp32
# or bf16 bits with "x_dtype"), the fp32 weight matrix ("w") and the sizes.
# ----------------------------------------------------------------------------

def tiny(seed: int = 0) -> dict:
    """Single BitLinear: X fp32 [8, 256] N(0,1), 1 % entries x20; W [256, 256]."""
    rng = np.random.default_rng(seed)
    x = add_entry_outliers(rng, gaussian(rng, (8, 256)), 0.01, 20.0)
    return dict(name="tiny_bitlinear_m8_k256_n256", x=x, x_dtype="f32",
                w=weights(256, 256, seed), M=8, K=256, N=256, act_bits=8)


def decode(M: int = 16, seed: int = 0, with_weights: bool = True) -> dict:
    """Decode GEMV: X bf16 [M, 2560] N(0,1), 0.5 % entries x30; W [6912, 2560]."""
    rng = np.random.default_rng(seed)
    x = add_entry_outliers(rng, gaussian(rng, (M, 2560)), 0.005, 30.0)
    return dict(name=f"decode_gemv_m{M}_k2560_n6912", x=f32_to_bf16_bits(x), x_dtype="bf16",
                w=weights(6912, 2560, seed) if with_weights else None,
                M=M, K=2560, N=6912, act_bits=8)


def prefill(seed: int = 0, M: int = 4096, with_weights: bool = True) -> dict:
    """Prefill GEMM: X bf16 [4096, 4096] N(0,1), 0.5 % channels x30; W [11008, 4096]."""
    rng = np.random.default_rng(seed)
    x = add_channel_outliers(rng, gaussian(rng, (M, 4096)), 0.005, 30.0)
    return dict(name=f"prefill_gemm_m{M}_k4096_n11008", x=f32_to_bf16_bits(x), x_dtype="bf16",
                w=weights(11008, 4096, seed) if with_weights else None,
                M=M, K=4096, N=11008, act_bits=8)


def hbitlinear(seed: int = 0, M: int = 2048, with_weights: bool = True) -> dict:
    """H-BitLinear a4: X bf16 [2048, 8192] Student-t(3) + 0.5 % fixed channels x50."""
    rng = np.random.default_rng(seed)
    x = add_channel_outliers(rng, student_t(rng, (M, 8192), 3), 0.005, 50.0)
    return dict(name=f"hbitlinear_a4_m{M}_k8192_n2048", x=f32_to_bf16_bits(x), x_dtype="bf16",
                w=weights(2048, 8192, seed) if with_weights else None,
                M=M, K=8192, N=2048, act_bits=4, had_block=8192)


# Layer shapes of the stacked BitLinear chain (hidden 2048, FFN 5632).
CHAIN_HIDDEN = 2048
CHAIN_FFN = 5632
CHAIN_HEADS = 16
CHAIN_PROJ = (  # name, N (out), K (in), activation bits of its input
    ("q", 2048, 2048, 8), ("k", 2048, 2048, 8), ("v", 2048, 2048, 8),
    ("o", 2048, 2048, 4), ("up", 5632, 2048, 8), ("gate", 5632, 2048, 8),
    ("down", 2048, 5632, 4),
)


def chain_input(M: int, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return gaussian(rng, (M, CHAIN_HIDDEN))


def chain_weights(layer: int, seed: int = 0) -> dict:
    """fp32 N(0, 0.02) weights of one layer; each projection has its own stream."""
    out = {}
    for p, (name, N, K, _) in enumerate(CHAIN_PROJ):
        rng = np.random.default_rng([seed + WEIGHT_SEED_OFFSET, layer, p])
        out[name] = gaussian(rng, (N, K), 0.02)
    return out


def random_rows(M: int, K: int, seed: int, dtype: str = "bf16", scale: float = 1.0) -> np.ndarray:
    """Plain N(0, scale^2) activations for small parity sweeps."""
    rng = np.random.default_rng(seed)
    x = gaussian(rng, (M, K), scale)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x
