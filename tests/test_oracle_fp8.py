"""Pins of the oracle's FP8 (E4M3, per-tensor scale) W8A8 quantiser and of the
FP8 expert layer: E4M3 rounding against torch's float8_e4m3fn conversion (a
library routine), saturation, round trips, the error bound, the weight-scale
closed form, and the layer against a restatement built on torch's cast."""
import numpy as np
import pytest
import torch

from oracle import fp8 as F
from oracle import lmoe as O


def _torch_e4m3(x32: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 values through torch's float8_e4m3fn cast (in range)."""
    return torch.from_numpy(x32).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_quantize_matches_torch_cast_in_range():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-8, 4, 20000))).astype(np.float32)
    s = np.float32(0.37)
    r = np.float32(np.float32(1.0) / s)
    scaled = (x * r).astype(np.float32)
    inr = np.abs(scaled) <= 448.0
    got = F.fake_quant(x, s)
    want = _torch_e4m3(scaled) * np.float64(s)
    assert np.array_equal(got[inr], want[inr])
    assert inr.mean() > 0.9


def test_saturation_and_signed_zero():
    s = np.float32(0.5)
    x = np.array([1e6, -1e6, 224.0, 0.0, -0.0], dtype=np.float32)
    codes = F.quantize(x, s)
    assert codes[0] == 0x7E and codes[1] == 0xFE          # +-448
    assert codes[2] == 0x7E                                 # 224 / 0.5 = 448
    assert codes[3] == 0x00 and codes[4] == 0x80
    assert np.array_equal(F.fake_quant(x, s)[:3], [224.0, -224.0, 224.0])


def test_grid_values_round_trip_and_error_bound():
    s = np.float32(2.0 ** -5)
    grid = np.array([m * 2.0 ** e for e in range(-6, 9) for m in (1, 1.125, 1.25, 1.5, 1.875)
                     if m * 2.0 ** e <= 448], dtype=np.float64)
    x = (grid * s).astype(np.float32)
    assert np.array_equal(F.fake_quant(x, s), x.astype(np.float64))
    rng = np.random.default_rng(1)
    y = (rng.uniform(2.0 ** -6, 400, 5000) * s).astype(np.float32)
    err = np.abs(F.fake_quant(y, s) - y.astype(np.float64))
    # normal range: half a unit in the last of 3 mantissa bits
    assert np.all(err <= np.abs(y) * 2.0 ** -4 * (1 + 1e-6))


def test_weight_scale_closed_form():
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((64, 96)) * 0.02).astype(np.float32)
    s = F.weight_scale(W)
    assert s == np.float32(np.float32(np.abs(W).max()) / np.float32(448.0))
    codes = F.quantize(W, s)
    assert (codes & 0x7F).max() == 0x7E      # the largest magnitude maps to 448


def _restated_fp8_layer(p, K, s_u, s_h):
    """The FP8 expert layer restated with torch's float8 cast as quantiser and
    per-token loops (no oracle quantiser code)."""
    def fq(a, s):
        s32 = np.float32(s)
        r = np.float32(np.float32(1.0) / s32)
        return _torch_e4m3((np.asarray(a, np.float32) * r).astype(np.float32)) * np.float64(s32)

    def fqw(W):
        s = np.float32(np.float32(np.abs(W.astype(np.float32)).max()) / np.float32(448.0))
        return fq(W, s)

    x = p["x"]
    T = x.shape[0]
    sig = 1.0 / (1.0 + np.exp(-(x @ p["W_r"].T)))
    key = sig + p["b"]
    y = np.maximum(x @ p["W_s1"].T, 0) ** 2 @ p["W_s2"].T
    for t in range(T):
        top = sorted(range(len(key[t])), key=lambda e: (-key[t][e], e))[:K]
        ws = sig[t, top] / sig[t, top].sum()
        u = fq((p["W_dn"] @ x[t])[None, :], s_u)[0]
        v = np.zeros_like(u)
        for wk, e in zip(ws, top):
            g = fq((np.maximum(fqw(p["W1"][e]) @ u, 0) ** 2)[None, :], s_h)[0]
            v += wk * (fqw(p["W2"][e]) @ g)
        y[t] += p["W_upl"] @ v
    return y


def test_fp8_layer_matches_restatement_and_is_close_to_bf16():
    rng = np.random.default_rng(3)
    T, d, l, N, K, h, hs = 4, 32, 16, 6, 2, 16, 16
    p = dict(x=rng.standard_normal((T, d)), W_r=rng.standard_normal((N, d)) * 0.3,
             b=rng.standard_normal(N) * 0.1, W_dn=rng.standard_normal((l, d)) * 0.2,
             W1=rng.standard_normal((N, h, l)) * 0.2, W2=rng.standard_normal((N, l, h)) * 0.2,
             W_upl=rng.standard_normal((d, l)) * 0.2, W_s1=rng.standard_normal((hs, d)) * 0.2,
             W_s2=rng.standard_normal((d, hs)) * 0.2)
    for k in ("x", "W_dn", "W1", "W2"):        # weights as float32 values, as the GPU sees them
        p[k] = p[k].astype(np.float32).astype(np.float64)
    s_u, s_h = 0.02, 0.05
    quant = {"fmt": "fp8", "s_u": s_u, "s_h": s_h}
    out = O.layer_forward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: p["W1"][e],
                          lambda e: p["W2"][e], p["W_upl"], p["W_s1"], p["W_s2"], K, quant=quant)
    ref = _restated_fp8_layer(p, K, s_u, s_h)
    assert np.allclose(out["y"], ref, atol=1e-12, rtol=0)
    bf = O.layer_forward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: p["W1"][e],
                         lambda e: p["W2"][e], p["W_upl"], p["W_s1"], p["W_s2"], K)
    rel = np.sqrt(np.mean((out["r"] - bf["r"]) ** 2) / np.mean(bf["r"] ** 2))
    assert 0 < rel < 0.08


def test_w4a16_layer_quantises_weights_only():
    """W4A16: NVFP4 weights, activations untouched -- equal to the BF16 layer
    run on the NVFP4 images of W1 and W2."""
    from oracle import nvfp4 as Q
    rng = np.random.default_rng(5)
    T, d, l, N, K, h, hs = 4, 32, 32, 6, 2, 32, 16
    p = dict(x=rng.standard_normal((T, d)), W_r=rng.standard_normal((N, d)) * 0.3,
             b=np.zeros(N), W_dn=rng.standard_normal((l, d)) * 0.2,
             W1=rng.standard_normal((N, h, l)) * 0.2, W2=rng.standard_normal((N, l, h)) * 0.2,
             W_upl=rng.standard_normal((d, l)) * 0.2, W_s1=rng.standard_normal((hs, d)) * 0.2,
             W_s2=rng.standard_normal((d, hs)) * 0.2)
    out = O.layer_forward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: p["W1"][e],
                          lambda e: p["W2"][e], p["W_upl"], p["W_s1"], p["W_s2"], K,
                          quant={"fmt": "w4a16"})
    fq = lambda W: Q.fake_quant(W, Q.weight_global_scale(W))
    ref = O.layer_forward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: fq(p["W1"][e]),
                          lambda e: fq(p["W2"][e]), p["W_upl"], p["W_s1"], p["W_s2"], K)
    assert np.array_equal(out["y"], ref["y"])
    assert np.array_equal(out["u"], ref["u"])
