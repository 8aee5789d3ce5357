"""FP8 (E4M3) W8A8 expert path on the GPU against the oracle: the quantised
weights bit-exact, and the layer with identical quantisation within the
quantised-expert bar (max|err| <= 6e-2 RMS(y), as for NVFP4)."""
import numpy as np
import pytest
import torch

from lmoe_synth import CONFIGS
from oracle import fp8 as F

from _parity import check_segments_valid, compare_layer, compare_layer_pooled, make, quant_of

pytestmark = pytest.mark.gpu
TOL_Q = 6e-2


def test_fp8_weights_bit_exact():
    cfg = CONFIGS["tiny_fp8"]
    w, x, layer = make(cfg)
    for name, R, K in (("w1", cfg.h, cfg.l), ("w2", cfg.l, cfg.h)):
        codes = layer.debug(name + "q_codes").numpy()
        s = layer.debug(name + "q_g").numpy()
        assert codes.shape == (cfg.N * R, K)
        for e in range(cfg.N):
            We = w[name][e].float().cpu().numpy()
            se = F.weight_scale(We)
            assert s[e] == se
            assert np.array_equal(codes[e * R:(e + 1) * R], F.quantize(We, se)), (name, e)
    layer.close()


@pytest.mark.parametrize("T", [64, 37, 5])
def test_tiny_fp8_layer(T):
    cfg = CONFIGS["tiny_fp8"]
    w, x, layer = make(cfg, T=T)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    errs = compare_layer(layer, w, x, y, np.arange(T), cfg.K, tol=TOL_Q, quant=quant_of(cfg),
                         elem_rel=2.0 ** -7, check_v=False)
    print("tiny_fp8", T, errs)
    assert errs["v_rms_rel"] <= TOL_Q
    layer.close()


# 16 sampled tokens plus the first and last; the oracle quantises every
# touched expert matrix once, in a pool of processes (seconds per matrix)
@pytest.mark.parametrize("name,n", [("super_prefill_fp8", 16)])
def test_super_fp8_sampled_tokens(name, n):
    cfg = CONFIGS[name]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    check_segments_valid(layer, cfg.T, cfg.N, cfg.K)
    rng = np.random.default_rng(3000 + cfg.seed)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], rng.choice(cfg.T, n, replace=False)]))
    errs = compare_layer_pooled(layer, w, x, y, toks, cfg.K, tol=TOL_Q, quant=quant_of(cfg))
    print(name, errs)
    assert errs["v_rms_rel"] <= TOL_Q
    layer.close()
