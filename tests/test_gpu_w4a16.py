"""W4A16 expert path (NVFP4 weights expanded to f16 inside the GEMM, 16-bit
activations) on the GPU against the oracle's W4A16 layer.  W4A16 has NVFP4
weights, so the NVFP4 bar applies to y (max|err| <= 6e-2 RMS(y)); with the
weights quantised identically on both sides only 16-bit roundings remain,
and the experts' combined output v is held to 1e-2 RMS as well (measured:
y max error 1.9-2.1 % of RMS on the tiny layer, the BF16 path's level)."""
import numpy as np
import pytest
import torch

from lmoe_synth import CONFIGS

from _parity import check_segments_valid, compare_layer, make, quant_of

pytestmark = pytest.mark.gpu
TOL_Q = 6e-2      # NVFP4 bar on y
TOL_V_RMS = 1e-2  # RMS error of the experts' combined output


@pytest.mark.parametrize("T,wq", [(64, "1d"), (37, "1d"), (5, "1d"), (64, "mse"), (64, "2d")])
def test_tiny_w4a16_layer(T, wq):
    cfg = CONFIGS["tiny_w4a16"].with_(wq=wq)
    w, x, layer = make(cfg, T=T)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    errs = compare_layer(layer, w, x, y, np.arange(T), cfg.K, tol=TOL_Q, quant=quant_of(cfg))
    print("tiny_w4a16", T, wq, errs)
    assert errs["v_rms_rel"] <= TOL_V_RMS
    layer.close()


def test_w4a16_weights_are_the_nvfp4_weights():
    """The same quantised weights as the NVFP4-expert layer (the W4A16 GEMM
    reads the NVFP4 codes and scale atoms)."""
    a_cfg = CONFIGS["tiny_w4a16"]
    b_cfg = a_cfg.with_(fmt="nvfp4")
    _, _, a = make(a_cfg)
    _, _, b = make(b_cfg)
    for k in ("w1q_codes", "w1q_sf", "w1q_g", "w2q_codes", "w2q_sf", "w2q_g"):
        assert torch.equal(a.debug(k), b.debug(k)), k
    a.close()
    b.close()


# few tokens: the oracle quantises every touched expert matrix (~1 s each)
def test_super_decode_w4a16_sampled_tokens():
    cfg = CONFIGS["super_decode_w4a16"]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    check_segments_valid(layer, cfg.T, cfg.N, cfg.K)
    toks = np.array([0, cfg.T - 1])
    errs = compare_layer(layer, w, x, y, toks, cfg.K, tol=TOL_Q, quant=quant_of(cfg))
    print("super_decode_w4a16", errs)
    assert errs["v_rms_rel"] <= TOL_V_RMS
    layer.close()
