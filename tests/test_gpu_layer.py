"""Parity of the CUDA layer (through the C ABI) with the float64 oracle."""
import numpy as np
import pytest
import torch

from lmoe_synth import CONFIGS
from oracle import lmoe as O

from _parity import (TOL_BF16, check_segments_valid, compare_layer, elem_ok, make, max_rel,
                     oracle_tokens, to64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    cfg = CONFIGS["tiny"]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    torch.cuda.synchronize()
    yield cfg, w, x, layer, y
    layer.close()


def test_tiny_all_tokens(tiny):
    cfg, w, x, layer, y = tiny
    errs = compare_layer(layer, w, x, y, np.arange(cfg.T), cfg.K)
    assert layer.sync_status() == 0
    print("tiny errors:", errs)


def test_tiny_segments_bit_exact(tiny):
    cfg, w, x, layer, y = tiny
    o = oracle_tokens(w, x, cfg.K)
    gi = layer.debug("topk_idx").numpy()
    if np.all(o["gap"] > 1e-3):
        assert np.array_equal(gi, o["S"])      # slot order too
    check_segments_valid(layer, cfg.T, cfg.N, cfg.K)
    if np.array_equal(np.sort(gi, 1), np.sort(o["S"], 1)):
        counts, offsets, perm, inv = O.segments(o["S"], cfg.N)
        assert np.array_equal(layer.debug("counts").numpy(), counts)
        assert np.array_equal(layer.debug("offsets").numpy(), offsets)
        if np.array_equal(gi, o["S"]):
            assert np.array_equal(layer.debug("perm").numpy(), perm)
            assert np.array_equal(layer.debug("inv").numpy(), inv)


def test_tiny_logits_match(tiny):
    cfg, w, x, layer, y = tiny
    o = oracle_tokens(w, x, cfg.K)
    z = layer.debug("logits").numpy().astype(np.float64)
    assert np.max(np.abs(z - o["z"])) <= 1e-4 * max(1.0, np.abs(o["z"]).max())


@pytest.mark.parametrize("T", [1, 5, 16, 17, 33, 63])
def test_tiny_ragged_token_counts(tiny, T):
    cfg, w, x, layer, _ = tiny
    xs = x[:T].contiguous()
    y = layer.forward(xs)
    torch.cuda.synchronize()
    compare_layer(layer, w, xs, y, np.arange(T), cfg.K)


def test_deterministic(tiny):
    cfg, w, x, layer, _ = tiny
    a = layer.forward(x).clone()
    b = layer.forward(x).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_zero_tokens_is_noop(tiny):
    cfg, w, x, layer, _ = tiny
    y = layer.forward(x[:0])
    assert y.shape == (0, cfg.d)


def test_too_many_tokens_rejected(tiny):
    from latent_space_mixture_b200 import LmoeError
    cfg, w, x, layer, _ = tiny
    with pytest.raises(LmoeError) as e:
        layer.forward(torch.cat([x, x]))
    assert e.value.code == -1


def test_routed_branch_alone():
    """W_s2 = 0: y is the routed branch r = W_upl v alone."""
    cfg = CONFIGS["tiny"]
    w, x, layer = make(cfg, overrides={"w_s2": torch.zeros_like})
    y = layer.forward(x)
    o = oracle_tokens(w, x, cfg.K)
    assert np.all(o["sh"] == 0)
    ok, ratio, rr = elem_ok(to64(y), o["r"])
    assert ok, (ratio, rr)
    layer.close()


def test_shared_branch_alone():
    """W1 = 0: the experts give 0 and y is the shared expert alone."""
    cfg = CONFIGS["tiny"]
    w, x, layer = make(cfg, overrides={"w1": torch.zeros_like})
    y = layer.forward(x)
    o = oracle_tokens(w, x, cfg.K)
    assert np.all(o["r"] == 0)
    assert np.all(to64(layer.debug("v")) == 0)
    ok, ratio, rr = elem_ok(to64(y), o["sh"])
    assert ok, (ratio, rr)
    assert max_rel(to64(y), o["sh"]) <= TOL_BF16
    layer.close()


def test_single_expert_dense_ffn():
    """N=32 experts but a router that always picks expert 0 with K=1: the layer
    is the dense FFN W_upl W2[0] sqrelu(W1[0] W_dn x) + shared."""
    cfg = CONFIGS["tiny"].with_(K=1)
    bias = lambda b: torch.where(torch.arange(cfg.N, device=b.device) == 0,  # noqa: E731
                                 torch.full_like(b, 10.0), torch.zeros_like(b))
    w, x, layer = make(cfg, overrides={"router_bias": bias})
    y = layer.forward(x)
    assert np.all(layer.debug("topk_idx").numpy() == 0)
    assert np.all(layer.debug("topk_w").numpy() == 1.0)
    xx = to64(x)
    u = xx @ to64(w["w_dn"]).T
    dense = np.maximum(u @ to64(w["w1"][0]).T, 0) ** 2 @ to64(w["w2"][0]).T @ to64(w["w_upl"]).T
    shared = np.maximum(xx @ to64(w["w_s1"]).T, 0) ** 2 @ to64(w["w_s2"]).T
    assert max_rel(to64(y), dense + shared) <= TOL_BF16
    layer.close()


def test_forward_host_matches_device(tiny):
    cfg, w, x, layer, _ = tiny
    y_dev = layer.forward(x).cpu()
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    layer.forward_host(xh, yh)
    assert torch.equal(yh, y_dev)


# ---------------------------------------------------------------- full sizes


def _sample(T, n, seed):
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(T, size=min(n, T), replace=False))


@pytest.fixture(scope="module")
def super_decode():
    cfg = CONFIGS["super_decode"]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    torch.cuda.synchronize()
    yield cfg, w, x, layer, y
    layer.close()
    del w
    torch.cuda.empty_cache()


def test_super_decode_sampled_tokens(super_decode):
    cfg, w, x, layer, y = super_decode
    errs = compare_layer(layer, w, x, y, _sample(cfg.T, 24, 1001), cfg.K)
    print("super_decode errors:", errs)
    check_segments_valid(layer, cfg.T, cfg.N, cfg.K)
    assert layer.sync_status() == 0


@pytest.mark.parametrize("name,n", [("super_prefill", 16), ("ultra", 16)])
def test_large_configs_sampled_tokens(name, n):
    cfg = CONFIGS[name]
    w, x, layer = make(cfg)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    counts = check_segments_valid(layer, cfg.T, cfg.N, cfg.K)
    if cfg.bias == "zipf":
        assert (counts == 0).any(), "Zipf router bias leaves some experts without tokens"
    # sample includes the first and last token (first and last tiles)
    toks = np.unique(np.concatenate([[0, cfg.T - 1], _sample(cfg.T, n, 1000 + cfg.seed)]))
    errs = compare_layer(layer, w, x, y, toks, cfg.K)
    print(name, "errors:", errs)
    layer.close()
    del w, x, y
    torch.cuda.empty_cache()


def test_cta_pair_gemms_match_single_cta_gemms(monkeypatch):
    """The CTA-pair GEMMs (M=256 over two SMs, used at large token counts) and
    the single-CTA GEMMs give the same layer, and both match the oracle."""
    cfg = CONFIGS["pair_small"]
    monkeypatch.setenv("LMOE_PAIR", "0")
    w, x, single = make(cfg)
    y1 = single.forward(x).clone()
    monkeypatch.setenv("LMOE_PAIR", "1")
    from lmoe_synth import act_global_scales  # noqa: F401
    from latent_space_mixture_b200 import LatentMoE
    pair = LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, cfg.T, w)
    y2 = pair.forward(x)
    torch.cuda.synchronize()
    assert pair.sync_status() == 0 and single.sync_status() == 0
    assert max_rel(to64(y2), to64(y1)) <= 1e-2
    toks = np.unique(np.concatenate([[0, cfg.T - 1], _sample(cfg.T, 24, 9)]))
    errs = compare_layer(pair, w, x, y2, toks, cfg.K)
    print("pair_small errors:", errs)
    single.close()
    pair.close()


def test_split_k_pair_dense_gemms_match_single_cta(monkeypatch):
    """At decode-sized batches (one block of <= 256 tokens) the x- and
    y-GEMMs run on CTA pairs with K split into slices (fp32 partials summed
    by the split-K reductions); the layer matches the single-CTA split-K one
    (within 1e-2 of RMS(y): near-tie tokens may route apart) and the
    oracle."""
    cfg = CONFIGS["pair_small"]
    monkeypatch.setenv("LMOE_PAIR", "0")
    w, x, single = make(cfg, T=256)
    y1 = single.forward(x).clone()
    monkeypatch.setenv("LMOE_PAIR", "1")
    from latent_space_mixture_b200 import LatentMoE
    pair = LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, 256, w)
    y2 = pair.forward(x)
    torch.cuda.synchronize()
    assert pair.sync_status() == 0 and single.sync_status() == 0
    assert max_rel(to64(y2), to64(y1)) <= 1e-2
    toks = np.unique(np.concatenate([[0, 255], _sample(256, 24, 11)]))
    errs = compare_layer(pair, w, x, y2, toks, cfg.K)
    print("split-K pair errors:", errs)
    single.close()
    pair.close()


def test_segment_builders_agree_across_the_one_block_limit():
    """Up to 256 tokens the forward builds the per-expert segments in one
    block, above it with histogram, scan and scatter: on either side of the
    limit (255, 256, 257 tokens of the same batch, one handle) the segments
    hold the stable order exactly and each forward matches the oracle (the
    dense GEMMs' split-K plans change with T, so the three outputs agree
    within the oracle bar, not bit for bit)."""
    cfg = CONFIGS["pair_small"]
    w, x, layer = make(cfg, T=257)
    assert layer.launches_per_forward(256) == layer.launches_per_forward(257) - 2
    ys = {}
    for T in (255, 256, 257):
        xs = x[:T].contiguous()
        y = layer.forward(xs).clone()
        torch.cuda.synchronize()
        assert layer.sync_status() == 0
        check_segments_valid(layer, T, cfg.N, cfg.K)
        toks = np.unique(np.concatenate([[0, T - 1], _sample(T, 12, 29)]))
        compare_layer(layer, w, xs, y, toks, cfg.K)
        ys[T] = (y, np.sort(layer.debug("topk_idx").numpy(), axis=1))
    y0, s0 = ys[255]
    for T in (256, 257):
        y1, s1 = ys[T]
        same = np.all(s1[:255] == s0, axis=1)   # near-tie tokens may route apart
        assert same.mean() > 0.95
        rows = torch.from_numpy(np.nonzero(same)[0]).to(y0.device)
        assert max_rel(to64(y1[:255][rows]), to64(y0[rows])) <= 2 * TOL_BF16
    layer.close()


def test_overlapped_shared_expert_matches_serial_forward(monkeypatch):
    """The forward that runs the shared expert's GEMMs on a side stream over
    a share of the SMs (opt-in, LMOE_OVERLAP; forced here) equals the serial
    forward within the oracle bar, and matches the oracle."""
    cfg = CONFIGS["pair_small"]
    monkeypatch.setenv("LMOE_OVERLAP", "0")
    w, x, layer = make(cfg)
    y0 = layer.forward(x).clone()
    assert layer.launches_per_forward(cfg.T) == 10
    monkeypatch.setenv("LMOE_OVERLAP", "16")
    assert layer.launches_per_forward(cfg.T) == 12
    y1 = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    # both bf16 outputs within 2e-2 RMS(y) of the oracle: within twice that
    # of each other
    assert max_rel(to64(y1), to64(y0)) <= 2 * 2e-2
    toks = np.unique(np.concatenate([[0, cfg.T - 1], _sample(cfg.T, 24, 19)]))
    errs = compare_layer(layer, w, x, y1, toks, cfg.K)
    print("overlapped pair_small errors:", errs)
    layer.close()
