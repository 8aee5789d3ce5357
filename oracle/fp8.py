"""FP8 (E4M3) W8A8 quantiser of the oracle for the expert GEMMs.

TEST INFRASTRUCTURE ONLY (see oracle/lmoe.py).  Shares no code with the CUDA
library.

Source: "Nemotron-3 Super 精读报告", section 9.1 (FP8 checkpoint): the MoE
GEMMs run in FP8 with both weights and activations quantised (W8A8).  The
page gives the checkpoint's precision per component, not the scaling.

Readings:
  * the element format is E4M3 (the 'fn' variant: bias 7, no infinities,
    largest finite 448), rounded to nearest, ties to even, saturating;
  * one float32 scale per tensor: a weight matrix W[e] has
    s_W = amax(W[e]) / 448; the expert inputs u and the expert hidden
    activation use static per-layer scales s_u, s_h given with the weights
    (as the NVFP4 path's global scales);
  * arithmetic in IEEE float32 in this order: r = f32(1 / s) once per
    tensor, code = e4m3(f32(x * r)); value = code * s (a zero scale gives
    zero codes);
  * within this build the routed experts are FP8; the router, the latent
    projections and the shared expert stay BF16 (the pages' checkpoint also
    runs the shared expert in FP8; here it shares BF16 GEMMs with the router
    and the projections).
"""
from __future__ import annotations

import numpy as np

from .nvfp4 import e4m3_decode, e4m3_rtne

__all__ = ["E4M3_MAX", "weight_scale", "quantize", "fake_quant"]

E4M3_MAX = 448.0


def weight_scale(W: np.ndarray) -> np.float32:
    """s_W = amax(W) / 448 in float32."""
    amax = np.float32(np.max(np.abs(np.asarray(W, dtype=np.float32))))
    return np.float32(amax / np.float32(E4M3_MAX))


def quantize(X: np.ndarray, s) -> np.ndarray:
    """E4M3 codes (uint8) of X under the per-tensor scale s."""
    Xf = np.asarray(X, dtype=np.float32)
    s32 = np.float32(s)
    r = np.float32(np.float32(1.0) / s32) if s32 > 0 else np.float32(0.0)
    return e4m3_rtne((Xf * r).astype(np.float32))


def fake_quant(X: np.ndarray, s) -> np.ndarray:
    """Quantise-dequantise image of X (float64): code * s."""
    return e4m3_decode(quantize(X, s)) * np.float64(np.float32(s))
