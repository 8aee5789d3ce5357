"""NVFP4 gradient-path pieces of the oracle: the random Hadamard transform on
16-element blocks, and stochastic rounding of values to NVFP4.

TEST INFRASTRUCTURE ONLY (see oracle/lmoe.py).  Shares no code with the CUDA
library.

Source: "Nemotron-3 Super 精读报告", section 5.3 (NVFP4 格式细节): gradients
and activations are quantised with 1D blocks along the GEMM reduction axis, a
random Hadamard transform (RHT) is applied to the inputs of the weight-
gradient GEMMs, and stochastic rounding to the gradient tensors; section 9.3:
stochastic rounding is unbiased in expectation, trading the systematic drift
of round-to-nearest for zero-mean noise.  The pages give neither the
transform's size nor the generator of the random bits for these tensors.

Readings:
  * RHT: every 16-element block x_b of a row (the reduction axis) becomes
    y_b = (1/4) H16 (s * x_b), H16 the 16 x 16 Sylvester Hadamard matrix
    (entries +-1, so H16 / 4 is orthonormal and its own inverse) and s a
    vector of 16 signs drawn from a seed, shared by all blocks.  Arithmetic
    in float32 as a fast Walsh-Hadamard transform: stages h = 1, 2, 4, 8,
    each pair (i, i + h) with bit h of i clear becoming (a + b, a - b), then
    the product by 0.25 (exact).  The block size is that of the NVFP4
    micro-block (16).
  * random bits: a counter-based generator, SplitMix64 (G. Steele, D. Lea,
    C. Flood, "Fast splittable pseudorandom number generators", OOPSLA
    2014): for counter i, z = seed + (i + 1) * 0x9E3779B97F4A7C15 (mod 2^64),
    then z ^= z >> 30, z *= 0xBF58476D1CE4E5B9, z ^= z >> 27,
    z *= 0x94D049BB133111EB, z ^= z >> 31.  Element (row, col) of a
    [rows][cols] tensor takes counter row * cols + col; the RHT signs take
    counters 0..15 of the transform's seed (sign -1 when bit 63 is set).  A
    uniform number u in [0, 1) is the top 24 bits times 2^-24.
  * stochastic rounding to E2M1: the block scale is the round-to-nearest
    one of oracle.nvfp4 (s_b = E4M3(amax / (6 g)), r = f32(1 / (s_b g))) and
    v = f32(x * r); |v| >= 6 gives 6; otherwise lo <= |v| < hi are adjacent
    grid magnitudes and the code is hi when u < p = (|v| - lo) / (hi - lo),
    else lo (p is exact in float32: hi - lo is a power of two and
    |v| - lo is exact); the sign bit follows v.  So E[q] = v on [0, 6].
"""
from __future__ import annotations

import numpy as np

from .nvfp4 import E2M1_GRID, _block_scales, e2m1_decode, e4m3_decode

__all__ = ["splitmix64", "uniform24", "rht_signs", "rht16", "e2m1_sr", "quantize_sr",
           "fake_quant_sr"]

BLOCK = 16
_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, counters: np.ndarray) -> np.ndarray:
    """SplitMix64 output for each counter (uint64 array)."""
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed) + (c + np.uint64(1)) * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform24(seed: int, counters: np.ndarray) -> np.ndarray:
    """Uniform float32 numbers in [0, 1): the top 24 bits times 2^-24."""
    top = (splitmix64(seed, counters) >> np.uint64(40)).astype(np.float64)
    return (top * 2.0 ** -24).astype(np.float32)


def rht_signs(seed: int) -> np.ndarray:
    """The transform's 16 signs (float32 +-1)."""
    bits = splitmix64(seed, np.arange(BLOCK, dtype=np.uint64)) >> np.uint64(63)
    return np.where(bits == 1, np.float32(-1.0), np.float32(1.0)).astype(np.float32)


def rht16(X: np.ndarray, seed: int = None, signs: np.ndarray = None) -> np.ndarray:
    """(1/4) H16 (s * x) on every 16-element block of the last axis, float32
    butterflies in the order of the module docstring."""
    Xf = np.asarray(X, dtype=np.float32)
    if Xf.shape[-1] % BLOCK:
        raise ValueError("last axis must be a multiple of 16")
    s = rht_signs(seed) if signs is None else np.asarray(signs, dtype=np.float32)
    b = (Xf.reshape(-1, BLOCK) * s[None, :]).astype(np.float32)
    h = 1
    while h < BLOCK:
        out = b.copy()
        for i in range(BLOCK):
            if i & h:
                continue
            a, c = b[:, i], b[:, i + h]
            out[:, i] = (a + c).astype(np.float32)
            out[:, i + h] = (a - c).astype(np.float32)
        b = out
        h *= 2
    return (b * np.float32(0.25)).astype(np.float32).reshape(Xf.shape)


def e2m1_sr(v: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Stochastic rounding of float32 values v to E2M1 codes with uniforms u."""
    v = np.asarray(v, dtype=np.float32)
    u = np.asarray(u, dtype=np.float32)
    mag = np.abs(v)
    lo = np.clip(np.searchsorted(E2M1_GRID, mag.astype(np.float64), side="right") - 1, 0, 6)
    lo_v = E2M1_GRID[lo].astype(np.float32)
    hi_v = E2M1_GRID[lo + 1].astype(np.float32)
    p = ((mag - lo_v) / (hi_v - lo_v)).astype(np.float32)
    code = np.where(u < p, lo + 1, lo)
    code = np.where(mag >= np.float32(6.0), 7, code)
    sign = np.signbit(v).astype(np.int64)
    return (code + 8 * sign).astype(np.uint8)


def quantize_sr(X: np.ndarray, g, seed: int) -> tuple:
    """NVFP4 of X [rows][cols] (cols a multiple of 16) with stochastically
    rounded elements.  Returns (codes uint8 [rows][cols], scale codes uint8
    [rows][cols/16], decoded scales float32 [rows][cols/16])."""
    Xf = np.asarray(X, dtype=np.float32)
    if Xf.ndim != 2 or Xf.shape[1] % BLOCK:
        raise ValueError("need [rows][cols], cols a multiple of 16")
    rows, cols = Xf.shape
    g32 = np.float32(g)
    blocks = Xf.reshape(-1, BLOCK)
    sc = _block_scales(blocks, g32, mse=False)
    sb = e4m3_decode(sc).astype(np.float32)
    denom = (sb * g32).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        rcp = (np.float32(1.0) / denom).astype(np.float32)
    rcp = np.where(denom > 0, rcp, np.float32(0.0)).astype(np.float32)
    v = (blocks * rcp[:, None]).astype(np.float32).reshape(rows, cols)
    u = uniform24(seed, np.arange(rows * cols, dtype=np.uint64)).reshape(rows, cols)
    codes = e2m1_sr(v, u)
    return codes, sc.reshape(rows, cols // BLOCK), sb.reshape(rows, cols // BLOCK)


def fake_quant_sr(X: np.ndarray, g, seed: int) -> np.ndarray:
    """Quantise-dequantise image (float64) of quantize_sr."""
    codes, _, sb = quantize_sr(X, g, seed)
    rows, cols = codes.shape
    q = e2m1_decode(codes).reshape(rows, cols // BLOCK, BLOCK)
    return (q * sb.astype(np.float64)[..., None] * np.float64(np.float32(g))).reshape(rows, cols)
