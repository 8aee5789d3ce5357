"""The pooled oracle of the quantised full-size parity tests equals the
oracle's layer_forward (CPU, tiny quantised layers)."""
import numpy as np
import pytest

from lmoe_synth import CONFIGS, make_weights, make_x
from tests._parity import oracle_tokens, oracle_tokens_pooled, quant_of


@pytest.mark.parametrize("name", ["tiny_fp8", "tiny_nvfp4", "tiny_w4a16"])
def test_pooled_oracle_equals_layer_forward(name):
    cfg = CONFIGS[name]
    w, gen = make_weights(cfg)
    x = make_x(cfg, gen, T=12)
    quant = quant_of(cfg)
    ref = oracle_tokens(w, x, cfg.K, quant=quant)
    got = oracle_tokens_pooled(w, x, cfg.K, quant, ref["S"], workers=3)
    for k in ("v", "y", "u", "hs", "w"):
        assert np.allclose(got[k], ref[k], atol=1e-12, rtol=0), k
