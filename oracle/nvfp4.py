"""NVFP4 quantiser of the oracle (E2M1 elements, 16-element micro-blocks,
E4M3 block scales, FP32 global scale).

TEST INFRASTRUCTURE ONLY (see oracle/lmoe.py).  Shares no code with the CUDA
library.

Sources:
  [R1] "NVIDIA Nemotron 3: Efficient and Open Intelligence" (xllm-io paper
       review), section 三 "NVFP4 训练": 16-element micro-block scaling, E4M3
       block scale factors, a second-level FP32 global scale, E2M1 elements.
  [R5] "Nemotron-3 Super 精读报告", section 5.3 (NVFP4 格式细节): activations
       use 1D blocks along the GEMM reduction axis; section 9.2: activation
       block scales are max-based; table 5.2: latent projections stay BF16.
  [R5] section 9.3 names round-to-nearest, ties to even (RTNE) as the
       standard rounding (stochastic rounding is used only for the SSM cache).

Readings (the pages fix the format, not the scale arithmetic):
  * blocks are 16 consecutive elements along the last axis, which the caller
    makes the GEMM reduction axis;
  * block scale s_b = E4M3_rtne_satfinite(amax_b / (6 g)), element
    q = E2M1_rtne_satfinite(x * r_b) with r_b = 1 / (s_b g) rounded once
    per block (a reciprocal per block rather than a division per element),
    value q * s_b * g;
  * a weight matrix's global scale is g_W = amax(W) / (6 * 448);
  * all scale and element arithmetic is IEEE float32 in exactly this order,
    so that two implementations of it produce identical codes:
        six_g = f32(6 * g); sbf = f32(amax / six_g); s_b = e4m3(sbf);
        denom = f32(s_b * g); r = f32(1 / denom), or 0 when denom == 0;
        q = e2m1(f32(x * r)) (a zero-scale block gives +-0 codes);
  * weights use the same 1D max-based blocks as activations (the pages'
    training recipe uses 2D weight blocks and their PTQ an MSE search; both
    are left out of this oracle).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "E2M1_GRID", "e2m1_rtne", "e2m1_decode", "e4m3_rtne", "e4m3_decode",
    "e4m3_value", "weight_global_scale", "quantize", "fake_quant", "BLOCK",
]

BLOCK = 16
# E2M1 magnitudes, indexed by the 3-bit code (exponent 2 bits, mantissa 1 bit,
# exponent bias 1, subnormal at exponent 0)
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E4M3_MAX = 448.0


def e2m1_rtne(x: np.ndarray) -> np.ndarray:
    """Round float values to E2M1 codes (uint8 0..15, bit 3 = sign).

    Nearest grid magnitude, ties to the even code (mantissa bit 0), magnitudes
    at or above 6 saturate to 6.  The sign bit follows the input's sign bit.
    """
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN has no E2M1 code")
    mag = np.abs(x)
    lo = np.clip(np.searchsorted(E2M1_GRID, mag, side="right") - 1, 0, 7)
    hi = np.minimum(lo + 1, 7)
    mid = 0.5 * (E2M1_GRID[lo] + E2M1_GRID[hi])
    up = (mag > mid) | ((mag == mid) & (lo % 2 == 1))
    code = np.where(up, hi, lo)
    code = np.where(mag >= 6.0, 7, code)
    sign = np.signbit(x).astype(np.int64)
    return (code + 8 * sign).astype(np.uint8)


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    v = E2M1_GRID[code & 7]
    return np.where(code & 8, -v, v)


def e4m3_rtne(x: np.ndarray) -> np.ndarray:
    """Round float values to E4M3 (the 'fn' variant: bias 7, no infinities,
    largest finite 448) codes, round-to-nearest-even, saturating to +-448."""
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN input")
    sign = np.signbit(x)
    a = np.abs(x)
    m, ex = np.frexp(a)                      # a = m 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)               # floor(log2 a), subnormals at -6
    quantum = np.ldexp(1.0, e - 3)           # 3 mantissa bits
    q = np.rint(a / quantum) * quantum       # rint: half to even
    q = np.where(a == 0, 0.0, q)
    q = np.minimum(q, E4M3_MAX)
    # encode
    m2, ex2 = np.frexp(q)
    E = np.where(q >= 2.0 ** -6, ex2 - 1 + 7, 0)
    mant = np.where(E > 0, np.rint((q / np.ldexp(1.0, E - 7) - 1.0) * 8.0),
                    np.rint(q / 2.0 ** -9))
    code = (E.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(q == 0, 0, code)
    return (code | (sign.astype(np.int64) << 7)).astype(np.uint8)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.int64)
    E = (code >> 3) & 15
    M = code & 7
    v = np.where(E == 0, M * 2.0 ** -9, (1.0 + M / 8.0) * np.ldexp(1.0, E - 7))
    if ((E == 15) & (M == 7)).any():
        raise ValueError("E4M3 NaN code")
    return np.where(code & 0x80, -v, v)


def e4m3_value(x: np.ndarray) -> np.ndarray:
    """E4M3 round-trip of x as float32 values."""
    return e4m3_decode(e4m3_rtne(x)).astype(np.float32)


def weight_global_scale(W: np.ndarray) -> np.float32:
    """g_W = amax(W) / (6 * 448) in float32 (second-level FP32 global scale)."""
    amax = np.float32(np.max(np.abs(np.asarray(W, dtype=np.float32))))
    return np.float32(amax / np.float32(6.0 * E4M3_MAX))


def quantize(X: np.ndarray, g) -> tuple:
    """NVFP4 codes of X along its last axis (a multiple of 16).

    Returns (codes uint8 [..., n] E2M1 codes, scale_codes uint8 [..., n/16]
    E4M3 codes, scales float32 [..., n/16] decoded block scales).
    """
    Xf = np.asarray(X, dtype=np.float32)
    n = Xf.shape[-1]
    if n % BLOCK:
        raise ValueError("last axis must be a multiple of 16")
    g32 = np.float32(g)
    blocks = Xf.reshape(Xf.shape[:-1] + (n // BLOCK, BLOCK))
    amax = np.max(np.abs(blocks), axis=-1)
    six_g = np.float32(np.float32(6.0) * g32)
    with np.errstate(divide="ignore", invalid="ignore"):
        sbf = (amax / six_g).astype(np.float32) if six_g > 0 else np.zeros_like(amax)
    sbf = np.where(np.isfinite(sbf), sbf, np.float32(0.0)).astype(np.float32)
    sc = e4m3_rtne(sbf)
    sb = e4m3_decode(sc).astype(np.float32)
    denom = (sb * g32).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        rcp = (np.float32(1.0) / denom).astype(np.float32)
    rcp = np.where(denom > 0, rcp, np.float32(0.0)).astype(np.float32)
    ratio = (blocks * rcp[..., None]).astype(np.float32)
    # a block whose scale is 0 gives x * 0 = +-0: value 0, sign kept (IEEE)
    codes = e2m1_rtne(ratio).astype(np.uint8)
    return codes.reshape(Xf.shape), sc, sb


def fake_quant(X: np.ndarray, g) -> np.ndarray:
    """Quantise-dequantise image of X (float64): q * s_b * g."""
    X = np.asarray(X)
    codes, _, sb = quantize(X, g)
    n = X.shape[-1]
    q = e2m1_decode(codes).reshape(X.shape[:-1] + (n // BLOCK, BLOCK))
    out = q * sb.astype(np.float64)[..., None] * np.float64(np.float32(g))
    return out.reshape(X.shape)
