"""Pins of the oracle's NVFP4 quantiser: exhaustive E2M1 codes and ties, E4M3
against torch's float8_e4m3fn conversion (a library routine), saturation,
round trips and the per-element error bound."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4 as Q


def test_format_fixture_matches_oracle(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "nvfp4_format.json")))
    assert g["micro_block"] == Q.BLOCK == 16
    assert g["element_format"] == "E2M1" and g["block_scale_format"] == "E4M3"
    assert g["default_rounding"] == "RTNE"


def test_e2m1_all_codes_round_trip():
    # E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; exponent 0 subnormal
    expected = []
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        mag = (m * 0.5) if e == 0 else (1 + m * 0.5) * 2.0 ** (e - 1)
        expected.append(-mag if s else mag)
    vals = Q.e2m1_decode(np.arange(16))
    assert np.array_equal(vals, np.array(expected))
    assert np.array_equal(np.abs(vals[:8]), [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    assert np.array_equal(Q.e2m1_rtne(vals), np.arange(16, dtype=np.uint8))


def test_e2m1_ties_to_even_and_saturation():
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in ties.items():
        assert Q.e2m1_decode(Q.e2m1_rtne(np.array([x])))[0] == want
        assert Q.e2m1_decode(Q.e2m1_rtne(np.array([-x])))[0] == -want
    off = {0.2: 0.0, 0.3: 0.5, 0.8: 1.0, 1.3: 1.5, 2.6: 3.0, 3.4: 3.0, 4.9: 4.0,
           5.1: 6.0, 6.0: 6.0, 7.0: 6.0, 1e30: 6.0}
    for x, want in off.items():
        assert Q.e2m1_decode(Q.e2m1_rtne(np.array([x])))[0] == want


def test_e2m1_is_nearest_grid_point_brute_force():
    rng = np.random.default_rng(0)
    x = rng.uniform(-7, 7, 20000)
    grid = np.concatenate([-Q.E2M1_GRID[::-1], Q.E2M1_GRID])
    got = Q.e2m1_decode(Q.e2m1_rtne(x))
    dist = np.abs(np.clip(x, -6, 6)[:, None] - grid[None, :]).min(axis=1)
    assert np.allclose(np.abs(np.clip(x, -6, 6) - got), dist, atol=0)


def test_e4m3_all_codes_match_torch():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    ours = Q.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    assert Q.e4m3_decode(np.array([0x7E]))[0] == 448.0
    # every finite code encodes back to itself (except -0 -> sign kept)
    assert np.array_equal(Q.e4m3_rtne(ours), codes)


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.uniform(0, 448, 20000), np.exp(rng.uniform(-14, 6, 20000)),
        # exact midpoints between neighbouring codes
        0.5 * (Q.e4m3_decode(np.arange(1, 126)) + Q.e4m3_decode(np.arange(2, 127))),
    ]).astype(np.float32)
    ours = Q.e4m3_decode(Q.e4m3_rtne(x))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturates():
    assert np.array_equal(Q.e4m3_decode(Q.e4m3_rtne(np.array([449.0, 464.0, 500.0, 1e9]))),
                          [448.0] * 4)


def test_quantize_round_trip_of_grid_values():
    # blocks whose elements are q * s * g with representable s come back exactly
    rng = np.random.default_rng(2)
    g = np.float32(0.25)
    s_codes = rng.integers(0x20, 0x70, size=(4, 8))
    s = Q.e4m3_decode(s_codes)
    q = Q.e2m1_decode(rng.integers(0, 16, size=(4, 8, 16)))
    q[..., 0] = 6.0                       # each block reaches the E2M1 max
    X = (q * s[..., None] * g).reshape(4, 128)
    out = Q.fake_quant(X, g)
    assert np.array_equal(out, X)


def test_quantize_error_bound_and_zero_blocks():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((64, 256)).astype(np.float32) * 3
    X[5, 16:32] = 0.0
    g = Q.weight_global_scale(X)
    codes, sc, sb = Q.quantize(X, g)
    out = Q.fake_quant(X, g)
    assert np.all(out[5, 16:32] == 0.0)
    step = sb.astype(np.float64) * np.float64(g)       # per block
    err = np.abs(out - X).reshape(64, 16, 16)
    # nearest-point rounding: |err| <= half the widest E2M1 gap (1.0) * s*g
    # plus the saturation excess of the block max (scale rounding)
    amax = np.abs(X).reshape(64, 16, 16).max(axis=2)
    sat_excess = np.maximum(amax - 6 * step, 0)
    assert np.all(err <= (1.0 * step + sat_excess)[..., None] + 1e-12)
    # with g = amax/2688 the largest block scale is 448 (E4M3 max)
    assert sb.max() <= 448.0
    assert abs(float(sb.max()) - 448.0) <= 16.0


def test_weight_global_scale_closed_form():
    W = np.array([[0.5, -2688.0], [1.0, 0.0]], dtype=np.float32)
    assert Q.weight_global_scale(W) == np.float32(1.0)
    W = np.zeros((3, 16), dtype=np.float32)
    assert Q.weight_global_scale(W) == 0.0
    codes, sc, sb = Q.quantize(W, 0.0)
    assert np.all(codes == 0) and np.all(sb == 0)


def test_fake_quant_layer_close_to_bf16_layer():
    """The NVFP4 layer differs from the unquantised layer by a few percent of
    the routed output (a sanity bound on the dequantised values)."""
    from oracle import lmoe as O
    rng = np.random.default_rng(4)
    T, d, l, N, K, h, hs = 16, 64, 32, 8, 2, 48, 64
    x = rng.standard_normal((T, d))
    W = lambda *s: rng.standard_normal(s) * 0.1
    W_r, W_dn, W1, W2 = W(N, d), W(l, d), W(N, h, l), W(N, l, h)
    W_upl, W_s1, W_s2 = W(d, l), W(hs, d), W(d, hs)
    su = 0.1 * np.sqrt(d)
    sa = 0.1 * np.sqrt(l) * su
    quant = {"g_u": 8 * su / 2688, "g_h": (8 * sa) ** 2 / 2688}
    a = O.layer_forward(x, W_r, None, W_dn, lambda e: W1[e], lambda e: W2[e],
                        W_upl, W_s1, W_s2, K)
    b = O.layer_forward(x, W_r, None, W_dn, lambda e: W1[e], lambda e: W2[e],
                        W_upl, W_s1, W_s2, K, quant=quant)
    rel = np.sqrt(np.mean((a["r"] - b["r"]) ** 2)) / np.sqrt(np.mean(a["r"] ** 2))
    assert 0.0 < rel < 0.25
    assert np.array_equal(a["sh"], b["sh"])


# ----------------------------------------------------------------------------
# weight-scale variants: 2D 16x16 blocks and MSE-searched block scales

def _f32(v):
    return np.float32(v)


def _e2m1_nearest(r: float) -> float:
    """Nearest E2M1 value to r by exhaustive search, ties to the even code,
    saturating at +-6 (independent of the oracle's searchsorted version)."""
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    mag = min(abs(r), 6.0)
    best = None
    for code, gv in enumerate(grid):
        dist = abs(mag - gv)
        if best is None or dist < best[0] or (dist == best[0] and code % 2 == 0):
            best = (dist, code, gv)
    return -best[2] if np.signbit(r) else best[2]


def _scalar_block_error(vals, code, g):
    """Squared error of one block under E4M3 scale `code`, in float32 scalar
    steps in element order (plain loops, no vector code)."""
    s = _f32(Q.e4m3_decode(np.array([code]))[0])
    denom = _f32(s * _f32(g))
    rcp = _f32(_f32(1.0) / denom) if denom > 0 else _f32(0.0)
    err = _f32(0.0)
    for x in vals:
        q = _e2m1_nearest(float(_f32(_f32(x) * rcp)))
        deq = _f32(_f32(q) * denom)
        d = _f32(_f32(x) - deq)
        err = _f32(err + _f32(d * d))
    return err


def _scalar_mse_code(vals, g):
    amax = max(abs(float(v)) for v in vals)
    six_g = _f32(_f32(6.0) * _f32(g))
    c0 = int(Q.e4m3_rtne(np.array([_f32(_f32(amax) / six_g)]))[0])
    if c0 == 0:
        return 0
    best_code, best_err = None, None
    for code in range(max(1, c0 - 8), min(126, c0 + 2) + 1):
        e = _scalar_block_error(vals, code, g)
        if best_err is None or e <= best_err:
            best_code, best_err = code, e
    return best_code


def test_2d_block_scale_is_the_16x16_amax():
    rng = np.random.default_rng(41)
    W = (rng.standard_normal((48, 64)) * 0.02).astype(np.float32)
    W[5, 17] = 0.5          # one large value: its 16x16 block's rows share it
    g = Q.weight_global_scale(W)
    codes, sc, sb = Q.quantize(W, g, block2d=True)
    for rg in range(3):
        for kb in range(4):
            blk = W[16 * rg:16 * rg + 16, 16 * kb:16 * kb + 16]
            want = Q.e4m3_rtne(np.array([_f32(_f32(np.abs(blk).max()) / _f32(6 * g))]))[0]
            assert np.all(sc[16 * rg:16 * rg + 16, kb] == want)
    # the rows sharing the large value get its scale, not their own
    assert sc[0, 1] == sc[15, 1] and sc[0, 1] > Q.quantize(W, g)[1][0, 1]
    # elements: the 1D quantiser's arithmetic under the shared scale
    for r in (0, 5, 31):
        for kb in range(4):
            denom = _f32(_f32(sb[r, kb]) * g)
            rcp = _f32(_f32(1.0) / denom)
            for j in range(16):
                want = _e2m1_nearest(float(_f32(W[r, 16 * kb + j] * rcp)))
                assert Q.e2m1_decode(codes[r:r + 1, 16 * kb + j])[0] == want


def test_2d_blocks_of_identical_rows_equal_1d_blocks():
    rng = np.random.default_rng(42)
    row = (rng.standard_normal((1, 64)) * 0.03).astype(np.float32)
    W = np.repeat(row, 32, axis=0)
    g = Q.weight_global_scale(W)
    a, b = Q.quantize(W, g, block2d=True), Q.quantize(W, g)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("block2d", [False, True])
def test_mse_scale_matches_scalar_brute_force(block2d):
    rng = np.random.default_rng(43 + block2d)
    W = (rng.standard_normal((32, 48)) * 0.02).astype(np.float32)
    W[3, 5] = 0.2            # outliers make smaller scales competitive
    W[20, 40] = -0.15
    g = Q.weight_global_scale(W)
    _, sc, _ = Q.quantize(W, g, block2d=block2d, mse=True)
    for r0 in range(0, 32, 16):
        for kb in range(3):
            if block2d:
                vals = W[r0:r0 + 16, 16 * kb:16 * kb + 16].reshape(-1)   # row-major
                assert np.all(sc[r0:r0 + 16, kb] == _scalar_mse_code(vals, g))
            else:
                for r in (r0, r0 + 3, r0 + 15):
                    vals = W[r, 16 * kb:16 * kb + 16]
                    assert sc[r, kb] == _scalar_mse_code(vals, g)


def test_mse_never_worse_than_max_based_and_keeps_grid_blocks():
    rng = np.random.default_rng(44)
    W = (rng.standard_normal((64, 128)) * 0.02).astype(np.float32)
    g = Q.weight_global_scale(W)
    f_max = Q.fake_quant(W, g)
    f_mse = Q.fake_quant(W, g, mse=True)
    e_max = ((W.astype(np.float64) - f_max) ** 2).reshape(-1, 16).sum(1)
    e_mse = ((W.astype(np.float64) - f_mse) ** 2).reshape(-1, 16).sum(1)
    assert np.all(e_mse <= e_max * (1 + 1e-5) + 1e-30)
    assert (e_mse < e_max * (1 - 1e-3)).any()
    # a block exactly on the E2M1 grid under its max-based scale keeps it
    s0 = _f32(Q.e4m3_decode(np.array([0x30]))[0])    # 2^(6-7) * 1 = 0.5
    gg = _f32(1.0 / 8)
    blk = np.array([6, -4, 3, 1.5, 0.5, 0, -6, 2, 1, -3, 4, 0.5, -1, 6, 2, -0.5],
                   dtype=np.float32) * _f32(s0 * gg)
    _, sc, _ = Q.quantize(blk[None, :], gg, mse=True)
    assert sc[0, 0] == 0x30
    assert np.array_equal(Q.fake_quant(blk[None, :], gg, mse=True)[0], blk.astype(np.float64))


# ----------------------------------------------------------------------------
# the NVFP4 expert layer: which tensors are quantised, along which axis, with
# which global scale ("Nemotron-3 Super 精读报告", section 5.3: E2M1 elements in
# 16-element micro-blocks along the GEMM reduction axis, E4M3 block scales, an
# FP32 global scale; table 5.2: the latent projections stay BF16)

def _torch_e4m3_value(v: np.float32) -> np.float32:
    """E4M3 value of a non-negative float32 through torch's float8_e4m3fn cast,
    saturating at 448 first (the cast itself has no saturation)."""
    v = min(float(v), 448.0)
    return _f32(torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn)
                .to(torch.float32).item())


def _restated_block_quant(vec, g) -> np.ndarray:
    """Quantise-dequantise one vector in 16-element blocks along it, scalar
    float32 steps: s = E4M3(amax / (6 g)), r = 1 / (s g) once per block,
    q = nearest E2M1 of x r (ties to even), value q s g."""
    g32 = _f32(g)
    six_g = _f32(_f32(6.0) * g32)
    out = []
    for b0 in range(0, len(vec), 16):
        blk = [_f32(v) for v in vec[b0:b0 + 16]]
        amax = max(abs(float(v)) for v in blk)
        s = _torch_e4m3_value(_f32(_f32(amax) / six_g)) if six_g > 0 else _f32(0.0)
        denom = _f32(s * g32)
        r = _f32(_f32(1.0) / denom) if denom > 0 else _f32(0.0)
        for v in blk:
            q = _e2m1_nearest(float(_f32(v * r)))
            out.append(q * float(s) * float(g32))
    return np.array(out)


def _restated_weight_quant(W) -> np.ndarray:
    """Each row of an expert matrix [out][in] in blocks along `in` (the GEMM
    reduction axis), global scale amax(W) / (6 * 448) of that matrix."""
    W32 = np.asarray(W, dtype=np.float32)
    amax = max(abs(float(v)) for v in W32.reshape(-1))
    g = _f32(_f32(amax) / _f32(2688.0))
    return np.stack([_restated_block_quant(row, g) for row in W32])


def _restated_nvfp4_layer(p, K, g_u, g_h):
    """The NVFP4 expert layer with per-token loops: u quantised with g_u, W1[e]
    and W2[e] with their own weight scales, sqrelu(W1 u) with g_h; the router,
    projections and shared expert unquantised.  Uses no oracle quantiser."""
    x = p["x"]
    T = x.shape[0]
    sig = 1.0 / (1.0 + np.exp(-(x @ p["W_r"].T)))
    key = sig + p["b"]
    y = np.maximum(x @ p["W_s1"].T, 0) ** 2 @ p["W_s2"].T
    v_all = np.zeros((T, p["W_dn"].shape[0]))
    for t in range(T):
        top = sorted(range(len(key[t])), key=lambda e: (-key[t][e], e))[:K]
        ws = sig[t, top] / sig[t, top].sum()
        u = _restated_block_quant(p["W_dn"] @ x[t], g_u)
        v = np.zeros_like(u)
        for wk, e in zip(ws, top):
            a = _restated_weight_quant(p["W1"][e]) @ u
            hq = _restated_block_quant(np.maximum(a, 0) ** 2, g_h)
            v += wk * (_restated_weight_quant(p["W2"][e]) @ hq)
        v_all[t] = v
        y[t] += p["W_upl"] @ v
    return y, v_all


def _small_nvfp4_layer():
    rng = np.random.default_rng(45)
    T, d, l, N, K, h, hs = 6, 32, 32, 6, 2, 48, 16     # l != h: the blocking axis shows
    p = dict(x=rng.standard_normal((T, d)), W_r=rng.standard_normal((N, d)) * 0.3,
             b=rng.standard_normal(N) * 0.05, W_dn=rng.standard_normal((l, d)) * 0.2,
             W1=rng.standard_normal((N, h, l)) * 0.2, W2=rng.standard_normal((N, l, h)) * 0.2,
             W_upl=rng.standard_normal((d, l)) * 0.2, W_s1=rng.standard_normal((hs, d)) * 0.2,
             W_s2=rng.standard_normal((d, hs)) * 0.2)
    for k in p:                      # weights and x as bf16 values, as the GPU sees them
        p[k] = torch.from_numpy(p[k]).to(torch.bfloat16).to(torch.float64).numpy()
    su = 0.2 * np.sqrt(d)
    sa = 0.2 * np.sqrt(l) * su
    # static scales, deliberately not power-of-two multiples of each other
    return p, K, 8 * su / 2688 * 1.13, (8 * sa) ** 2 / 2688 * 0.71


def _oracle_nvfp4(p, K, g_u, g_h):
    from oracle import lmoe as O
    return O.layer_forward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: p["W1"][e],
                           lambda e: p["W2"][e], p["W_upl"], p["W_s1"], p["W_s2"], K,
                           quant={"g_u": g_u, "g_h": g_h})


def test_nvfp4_layer_matches_loop_restatement():
    p, K, g_u, g_h = _small_nvfp4_layer()
    y_ref, v_ref = _restated_nvfp4_layer(p, K, g_u, g_h)
    out = _oracle_nvfp4(p, K, g_u, g_h)
    assert np.allclose(out["v"], v_ref, atol=1e-12, rtol=0)
    assert np.allclose(out["y"], y_ref, atol=1e-12, rtol=0)
    # the single-token path (used for near-tie tokens) quantises the same way
    from oracle import lmoe as O
    for t in (0, 5):
        one = O.token_forward(p["x"][t], out["S"][t], out["s"][t], p["W_dn"],
                              lambda e: p["W1"][e], lambda e: p["W2"][e], p["W_upl"],
                              quant={"g_u": g_u, "g_h": g_h})
        assert np.allclose(one["v"], v_ref[t], atol=1e-12, rtol=0)


@pytest.mark.parametrize("mistake", ["none", "hidden_unquantised", "g_u_for_hidden",
                                     "w2_blocked_along_latent", "one_scale_for_all_experts"])
def test_nvfp4_restatement_catches_planted_mistakes(monkeypatch, mistake):
    """Each plausible slip in the oracle's quantised composition, planted in
    the oracle on the CPU, moves its output off the restatement ("none": the
    same harness without a slip stays on it)."""
    from oracle import lmoe as O
    from oracle import nvfp4 as Qn
    p, K, g_u, g_h = _small_nvfp4_layer()
    y_ref, _ = _restated_nvfp4_layer(p, K, g_u, g_h)
    l, h = p["W2"].shape[1], p["W2"].shape[2]
    g_all = Qn.weight_global_scale(np.concatenate([p["W1"].reshape(-1), p["W2"].reshape(-1)]))

    def q_w(W):
        if mistake == "w2_blocked_along_latent" and W.shape == (l, h):
            return Qn.fake_quant(W.T, Qn.weight_global_scale(W)).T
        if mistake == "one_scale_for_all_experts":
            return Qn.fake_quant(W, g_all)
        return Qn.fake_quant(W, Qn.weight_global_scale(W))

    def quantisers(quant):
        q_u = lambda a: Qn.fake_quant(a, quant["g_u"])  # noqa: E731
        if mistake == "hidden_unquantised":
            q_h = lambda a: a  # noqa: E731
        elif mistake == "g_u_for_hidden":
            q_h = lambda a: Qn.fake_quant(a, quant["g_u"])  # noqa: E731
        else:
            q_h = lambda a: Qn.fake_quant(a, quant["g_h"])  # noqa: E731
        return q_u, q_w, q_h

    monkeypatch.setattr(O, "_expert_quantisers", quantisers)
    out = _oracle_nvfp4(p, K, g_u, g_h)
    if mistake == "none":
        assert np.allclose(out["y"], y_ref, atol=1e-12, rtol=0)
    else:
        assert np.max(np.abs(out["y"] - y_ref)) > 1e-9
