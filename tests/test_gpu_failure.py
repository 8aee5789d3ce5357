"""Failure paths on the GPU without a fault: a bounded device wait that runs out
reports TIMEOUT and leaves the context usable; bad arguments are rejected."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    from latent_space_mixture_b200 import lmoe_check_bounded_wait
    assert lmoe_check_bounded_wait(2_000_000) == -5       # 2 ms limit, TIMEOUT
    a = torch.ones(1000, device="cuda")
    assert float(a.sum().item()) == 1000.0


def test_layer_usable_after_timeout_probe():
    from latent_space_mixture_b200 import lmoe_check_bounded_wait
    from lmoe_synth import CONFIGS
    from _parity import compare_layer, make
    assert lmoe_check_bounded_wait(1_000_000) == -5
    cfg = CONFIGS["tiny"]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    assert layer.sync_status() == 0
    compare_layer(layer, w, x, y, np.arange(cfg.T), cfg.K)
    layer.close()


def test_bad_arguments():
    from latent_space_mixture_b200 import LatentMoE, LmoeError
    from lmoe_synth import CONFIGS, make_weights
    cfg = CONFIGS["tiny"]
    w, _ = make_weights(cfg, device="cuda")
    with pytest.raises(LmoeError) as e:
        LatentMoE(cfg.d, cfg.l, cfg.N, cfg.N + 1, cfg.h, cfg.hs, 64, w)   # K > N
    assert e.value.code == -1
    with pytest.raises(LmoeError) as e:
        LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, 64, w, expert_format="nvfp4")
    assert e.value.code == -2
    with pytest.raises(ValueError):
        LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h + 64, cfg.hs, 64, w)   # shape mismatch
