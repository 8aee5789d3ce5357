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
  [R5] section 5.3: the training recipe quantises weights with 2D blocks;
       section 9.2 (NVFP4 PTQ): weight block scales chosen by minimising
       the weight MSE, activation block scales max-based.

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
  * weights use the same 1D max-based blocks as activations by default;
    two weight variants follow the pages' other recipes:
      - 2D blocks (block2d): one scale per 16 x 16 block of a [rows][n]
        matrix (16 rows by 16 reduction elements), from the block's amax,
        shared by the 16 rows; elements as above;
      - MSE-searched scales (mse): the scale code of a block (1D or 2D) is
        the candidate with the smallest squared quantisation error, over
        the E4M3 codes from 8 below to 2 above the max-based code c0
        (clipped to the positive finite codes 1..126: down to about half
        and up to about 1.28 x the max-based scale); the error of a
        candidate is accumulated in float32 over the block's elements in
        row-major order, err = f32(err + f32(d * d)) with
        d = f32(x - f32(q_value * denom)); ties go to the higher code; an
        all-zero block keeps code 0.
    The search range and the float32 error order are this oracle's reading
    (the pages name the criterion, not the search).
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


MSE_CODES_BELOW, MSE_CODES_ABOVE = 8, 2


def _codes_for_scale(vals: np.ndarray, sc: np.ndarray, g32: np.float32):
    """E2M1 codes of the rows of `vals` ([B, m] float32) under the E4M3 scale
    codes sc [B], with the float32 scale arithmetic of the module docstring.
    Returns (codes [B, m], denom [B] float32)."""
    sb = e4m3_decode(sc).astype(np.float32)
    denom = (sb * g32).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        rcp = (np.float32(1.0) / denom).astype(np.float32)
    rcp = np.where(denom > 0, rcp, np.float32(0.0)).astype(np.float32)
    ratio = (vals * rcp[:, None]).astype(np.float32)
    # a block whose scale is 0 gives x * 0 = +-0: value 0, sign kept (IEEE)
    return e2m1_rtne(ratio).astype(np.uint8), denom


def _block_sq_error(vals: np.ndarray, codes: np.ndarray, denom: np.ndarray) -> np.ndarray:
    """float32 squared error of each block, summed in element order."""
    deq = (e2m1_decode(codes).astype(np.float32) * denom[:, None]).astype(np.float32)
    d = (vals - deq).astype(np.float32)
    err = np.zeros(vals.shape[0], dtype=np.float32)
    for j in range(vals.shape[1]):
        err = (err + (d[:, j] * d[:, j]).astype(np.float32)).astype(np.float32)
    return err


def _block_scales(vals: np.ndarray, g32: np.float32, mse: bool) -> np.ndarray:
    """E4M3 scale code of every block ([B, m] float32 values)."""
    amax = np.max(np.abs(vals), axis=-1)
    six_g = np.float32(np.float32(6.0) * g32)
    with np.errstate(divide="ignore", invalid="ignore"):
        sbf = (amax / six_g).astype(np.float32) if six_g > 0 else np.zeros_like(amax)
    sbf = np.where(np.isfinite(sbf), sbf, np.float32(0.0)).astype(np.float32)
    c0 = e4m3_rtne(sbf)
    if not mse:
        return c0
    best = c0.copy()
    best_err = np.full(vals.shape[0], np.inf, dtype=np.float32)
    base = c0.astype(np.int64)
    for k in range(-MSE_CODES_BELOW, MSE_CODES_ABOVE + 1):
        cand = np.clip(base + k, 1, 126).astype(np.uint8)
        codes, denom = _codes_for_scale(vals, cand, g32)
        err = _block_sq_error(vals, codes, denom)
        take = err <= best_err          # ascending codes: ties go to the higher
        best = np.where(take, cand, best)
        best_err = np.where(take, err, best_err)
    return np.where(base == 0, c0, best).astype(np.uint8)


def quantize(X: np.ndarray, g, block2d: bool = False, mse: bool = False) -> tuple:
    """NVFP4 codes of X along its last axis (a multiple of 16).

    block2d: X is [rows][n] with rows a multiple of 16 and each scale covers
    16 rows x 16 elements; mse: MSE-searched block scales (module docstring).
    Returns (codes uint8 [..., n] E2M1 codes, scale_codes uint8 [..., n/16]
    E4M3 codes, scales float32 [..., n/16] decoded block scales); with
    block2d the scale of a 2D block is repeated for each of its rows.
    """
    Xf = np.asarray(X, dtype=np.float32)
    n = Xf.shape[-1]
    if n % BLOCK:
        raise ValueError("last axis must be a multiple of 16")
    g32 = np.float32(g)
    if block2d:
        if Xf.ndim != 2 or Xf.shape[0] % BLOCK:
            raise ValueError("2D blocks need a [rows][n] matrix, rows a multiple of 16")
        rows = Xf.shape[0]
        # [row group][k block][16 rows][16 elements] -> one block per row of vals
        t = Xf.reshape(rows // BLOCK, BLOCK, n // BLOCK, BLOCK).transpose(0, 2, 1, 3)
        vals = np.ascontiguousarray(t).reshape(-1, BLOCK * BLOCK)
        sc2 = _block_scales(vals, g32, mse)                       # [groups * kblocks]
        sc = np.repeat(sc2.reshape(rows // BLOCK, 1, n // BLOCK), BLOCK, axis=1)
        sc = sc.reshape(rows, n // BLOCK)
    else:
        vals = Xf.reshape(-1, BLOCK)
        sc = _block_scales(vals, g32, mse).reshape(Xf.shape[:-1] + (n // BLOCK,))
    blocks = Xf.reshape(-1, BLOCK)
    codes, _ = _codes_for_scale(blocks, sc.reshape(-1), g32)
    sb = e4m3_decode(sc).astype(np.float32)
    return codes.reshape(Xf.shape), sc, sb


def fake_quant(X: np.ndarray, g, block2d: bool = False, mse: bool = False) -> np.ndarray:
    """Quantise-dequantise image of X (float64): q * s_b * g."""
    X = np.asarray(X)
    codes, _, sb = quantize(X, g, block2d=block2d, mse=mse)
    n = X.shape[-1]
    q = e2m1_decode(codes).reshape(X.shape[:-1] + (n // BLOCK, BLOCK))
    out = q * sb.astype(np.float64)[..., None] * np.float64(np.float32(g))
    return out.reshape(X.shape)
