"""The standard-MoE comparator (no latent projections: u = x, r = v) through
the same C ABI and kernels, against the float64 oracle's standard-MoE mode."""
import numpy as np
import pytest
import torch

from lmoe_synth import CONFIGS

from _parity import check_segments_valid, compare_layer, make, max_rel, to64

pytestmark = pytest.mark.gpu


def _sample(T, n, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(T, size=min(n, T), replace=False))


@pytest.fixture(scope="module")
def tiny_std():
    cfg = CONFIGS["tiny_std"]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    torch.cuda.synchronize()
    yield cfg, w, x, layer, y
    layer.close()


def test_tiny_std_all_tokens(tiny_std):
    cfg, w, x, layer, y = tiny_std
    assert "w_dn" not in w and "w_upl" not in w
    errs = compare_layer(layer, w, x, y, np.arange(cfg.T), cfg.K)
    check_segments_valid(layer, cfg.T, cfg.N, cfg.K)
    assert layer.sync_status() == 0
    print("tiny_std errors:", errs)


@pytest.mark.parametrize("T", [1, 7, 37, 63])
def test_tiny_std_ragged(tiny_std, T):
    cfg, w, x, layer, _ = tiny_std
    xs = x[:T].contiguous()
    y = layer.forward(xs)
    torch.cuda.synchronize()
    compare_layer(layer, w, xs, y, np.arange(T), cfg.K)


def test_tiny_std_has_no_latent_u(tiny_std):
    from latent_space_mixture_b200 import LmoeError
    layer = tiny_std[3]
    with pytest.raises(LmoeError):
        layer.debug("u")


def test_std_equals_latent_layer_with_identity_projections(tiny_std):
    """The same layer through the latent path with l = d and W_dn = W_upl = I
    (exact in bf16): routing and v identical, y equal up to the order of the
    final fp32 sums (one K loop over [v | hs] vs W_s2 hs plus v)."""
    cfg, w, x, layer, y = tiny_std
    from latent_space_mixture_b200 import LatentMoE
    eye = torch.eye(cfg.d, dtype=torch.bfloat16, device=x.device)
    wl = dict(w, w_dn=eye, w_upl=eye.clone())
    lat = LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, cfg.T, wl)
    y2 = lat.forward(x)
    y1 = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(lat.debug("topk_idx"), layer.debug("topk_idx"))
    assert torch.equal(lat.debug("v"), layer.debug("v"))
    assert torch.equal(lat.debug("hs"), layer.debug("hs"))
    assert max_rel(to64(y1), to64(y2)) <= 1e-2
    lat.close()


@pytest.mark.parametrize("name,n", [("std_decode", 24), ("std_prefill", 16)])
def test_std_configs_sampled_tokens(name, n):
    cfg = CONFIGS[name]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    counts = check_segments_valid(layer, cfg.T, cfg.N, cfg.K)
    if cfg.bias == "zipf":
        assert (counts == 0).any() or counts.max() > 4 * counts.mean()
    toks = np.unique(np.concatenate([[0, cfg.T - 1], _sample(cfg.T, n, 2000 + cfg.seed)]))
    errs = compare_layer(layer, w, x, y, toks, cfg.K)
    print(name, "errors:", errs)
    layer.close()
    del w
    torch.cuda.empty_cache()
