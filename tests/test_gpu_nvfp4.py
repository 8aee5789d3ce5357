"""NVFP4 expert path on the GPU against the oracle: the quantiser bit-exact,
the quantised weights bit-exact, and the layer with identical quantisation
within the NVFP4 bar (max|err| <= 6e-2 RMS(y))."""
from ctypes import c_float, c_void_p

import numpy as np
import pytest
import torch

from lmoe_synth import CONFIGS
from oracle import nvfp4 as Q

from _parity import (check_segments_valid, compare_layer, compare_layer_pooled, make, quant_of,
                     rms_rel, to64)

pytestmark = pytest.mark.gpu
TOL_NVFP4 = 6e-2


def _gpu_quantize(x: torch.Tensor, g: float):
    from latent_space_mixture_b200 import _lib
    lib = _lib.load()
    rows, cols = x.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=x.device)
    rc = lib.lmoe_nvfp4_quantize(c_void_p(x.data_ptr()), rows, cols, c_float(g),
                                 c_void_p(codes.data_ptr()), c_void_p(scales.data_ptr()),
                                 c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert rc == 0
    return codes.cpu().numpy(), scales.cpu().numpy()


def _unpack(codes_bytes):
    lo = codes_bytes & 0x0F
    hi = codes_bytes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes_bytes.shape[0], -1)


def test_quantizer_bit_exact_against_oracle():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((257, 512)) * np.exp(rng.uniform(-6, 6, (257, 1)))).astype(np.float32)
    x[3, :16] = 0.0                                   # an all-zero block
    x[4, :16] = -0.0
    x[5, 16:32] = rng.choice([0.25, 0.75, 1.25, 2.5, -5.0], 16)   # E2M1 ties at s*g = 1
    x[6, :] = 1e-30                                   # scale underflow
    g = float(np.float32(np.abs(x).max() / 2688.0))
    codes, scales = _gpu_quantize(torch.from_numpy(x).cuda(), g)
    oc, osc, _ = Q.quantize(x, g)
    assert np.array_equal(scales, osc)
    got = _unpack(codes)
    # +0 and -0 codes are both zero values; compare values and codes
    assert np.array_equal(Q.e2m1_decode(got), Q.e2m1_decode(oc))
    assert np.array_equal(got, oc)


def _weights_from_atoms(codes, atoms, rows, K, Kp):
    q = _unpack(codes)[:, :K]
    sc = np.empty((rows, K // 16), dtype=np.uint8)
    r = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    off = ((r // 128) * (Kp // 64) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    sc[:, :] = atoms[off]
    return q, sc


@pytest.mark.parametrize("wq", ["1d", "2d", "mse", "2d_mse"])
def test_quantised_weights_bit_exact(wq):
    cfg = CONFIGS["tiny_nvfp4"].with_(wq=wq)
    w, x, layer = make(cfg)
    opt = dict(block2d=wq in ("2d", "2d_mse"), mse=wq in ("mse", "2d_mse"))
    lp, hp = (cfg.l + 255) // 256 * 256, (cfg.h + 255) // 256 * 256
    for name, R, K, Kp in (("w1", cfg.h, cfg.l, lp), ("w2", cfg.l, cfg.h, hp)):
        codes = layer.debug(name + "q_codes").numpy()
        atoms = layer.debug(name + "q_sf").numpy()
        g = layer.debug(name + "q_g").numpy()
        q, sc = _weights_from_atoms(codes, atoms, cfg.N * R, K, Kp)
        for e in range(cfg.N):
            We = w[name][e].float().cpu().numpy()
            ge = Q.weight_global_scale(We)
            assert g[e] == ge
            oc, osc, _ = Q.quantize(We, ge, **opt)
            assert np.array_equal(sc[e * R:(e + 1) * R], osc), (name, e)
            assert np.array_equal(Q.e2m1_decode(q[e * R:(e + 1) * R]), Q.e2m1_decode(oc)), (name, e)
        # padding beyond K holds zero codes
        assert np.all(_unpack(codes)[:, K:] == 0)
    layer.close()


@pytest.mark.parametrize("T,wq", [(64, "1d"), (37, "1d"), (5, "1d"), (64, "2d"), (37, "mse"),
                                  (64, "2d_mse")])
def test_tiny_nvfp4_layer(T, wq):
    cfg = CONFIGS["tiny_nvfp4"].with_(wq=wq)
    w, x, layer = make(cfg, T=T)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    errs = compare_layer(layer, w, x, y, np.arange(T), cfg.K, tol=TOL_NVFP4, quant=quant_of(cfg),
                         elem_rel=2.0 ** -7, check_v=False)
    print("tiny_nvfp4", T, wq, errs)
    assert errs["v_rms_rel"] <= TOL_NVFP4
    layer.close()


def test_super_prefill_nvfp4_sampled_tokens():
    cfg = CONFIGS["super_prefill_nvfp4"]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    counts = check_segments_valid(layer, cfg.T, cfg.N, cfg.K)
    assert (counts == 0).any()
    rng = np.random.default_rng(1000 + cfg.seed)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], rng.choice(cfg.T, 16, replace=False)]))
    errs = compare_layer_pooled(layer, w, x, y, toks, cfg.K, tol=TOL_NVFP4, quant=quant_of(cfg))
    print("super_prefill_nvfp4", errs)
    assert errs["v_rms_rel"] <= TOL_NVFP4
    layer.close()


def test_quantised_weights_bit_exact_at_super_widths():
    """The 2D + MSE weight quantiser on Super-width expert matrices (l = 1024,
    h = 2688: many K blocks, 16-row groups across 128-row scale atoms), first
    and last expert (the oracle's MSE search costs seconds per matrix)."""
    cfg = CONFIGS["tiny_nvfp4"].with_(l=1024, h=2688, N=32, wq="2d_mse")
    w, x, layer = make(cfg)
    lp, hp = (cfg.l + 255) // 256 * 256, (cfg.h + 255) // 256 * 256
    for name, R, K, Kp in (("w1", cfg.h, cfg.l, lp), ("w2", cfg.l, cfg.h, hp)):
        codes = layer.debug(name + "q_codes").numpy()
        atoms = layer.debug(name + "q_sf").numpy()
        g = layer.debug(name + "q_g").numpy()
        q, sc = _weights_from_atoms(codes, atoms, cfg.N * R, K, Kp)
        for e in (0, cfg.N - 1):
            We = w[name][e].float().cpu().numpy()
            ge = Q.weight_global_scale(We)
            assert g[e] == ge
            oc, osc, _ = Q.quantize(We, ge, block2d=True, mse=True)
            assert np.array_equal(sc[e * R:(e + 1) * R], osc), (name, e)
            assert np.array_equal(Q.e2m1_decode(q[e * R:(e + 1) * R]), Q.e2m1_decode(oc)), (name, e)
    layer.close()


def test_activation_scale_tables_reproduce_the_division():
    """The activation quantisers of the NVFP4 layer take a block's scale code
    and the reciprocal of its denominator from tables instead of dividing.
    Pinned to the quantiser's definition (float32, oracle.nvfp4): threshold k
    is the smallest float amax whose code E4M3(f32(amax / f32(6 g))) is at
    least k (checked at the threshold and at the float just below it), and
    reciprocal k is f32(1 / f32(E4M3value(k) g))."""
    from lmoe_synth import act_global_scales
    cfg = CONFIGS["tiny_nvfp4"]
    w, x, layer = make(cfg)
    tab = layer.debug("scale_tables").numpy()
    for row, g in enumerate(act_global_scales(cfg)):
        g32 = np.float32(g)
        six_g = np.float32(np.float32(6.0) * g32)
        code = lambda a: int(Q.e4m3_rtne(np.array([np.float32(np.float32(a) / six_g)]))[0])  # noqa
        t = tab[row]
        assert t[0] == 0.0 and np.isinf(t[127])
        for k in range(1, 127):
            thr = np.float32(t[k])
            assert code(thr) >= k, (row, k)
            assert code(np.nextafter(thr, np.float32(0.0))) < k, (row, k)
            s = np.float32(Q.e4m3_decode(np.array([k]))[0])
            assert t[128 + k] == np.float32(np.float32(1.0) / np.float32(s * g32)), (row, k)
        assert t[128] == 0.0
        assert t[255] == np.float32(np.float32(1.0) / six_g)
    layer.close()
