"""GPU parity of the backward pass (lmoe_backward) and of the aux-loss-free
bias update (lmoe_bias_update) against the oracle (oracle.backward).

The oracle differentiates the float64 layer on the same bf16 weights, inputs
and upstream gradient, with the GPU's selected experts (where keys nearly tie,
either set is a correct forward; the backward follows the forward that ran).

Tolerance of every gradient G (derived from the arithmetic): the GPU path
rounds each intermediate gradient to bf16 (dv, w dv, dg -> da, du, dz and the
shared one), reads the saved bf16 activations (u, sqrelu(W1 u), v, hs) and
takes max(a, 0) as sqrt of the saved sqrelu(a); each rounding is <= 2^-9
relative, and a gradient carries about four of them in sequence.  So:
  * relative RMS error <= 1e-2 (~5 x 2^-9);
  * elementwise |err| <= 2^-7 |G| + 3e-2 RMS(G): the element's own chain of
    roundings (4 x 2^-9) plus the tail of the accumulated noise, the bf16
    error model of the forward's intermediates (tests/_parity.py).  A plain
    max|err| / RMS bar does not fit: an expert weight gradient is a sum over
    a handful of routed rows, heavy-tailed, with elements ~15 x its RMS.
The router gradient takes a difference of similar terms,
(dw_k - sum_j w_j dw_j), so its relative error is larger: relative RMS
<= 3e-2 and elementwise 2^-7 |G| + 8e-2 RMS(G).  An expert weight gradient
dW1[e] = sum_r da_r u_r^T (and dW2[e] likewise) sums only the expert's few
routed rows (8 on average in the tiny layer), of heavy-tailed factors
(da = dg 2 sqrt(g) is zero wherever the activation is, large elsewhere):
an element's error follows the magnitude of its few products, not of their
(partly cancelling) sum, and is not averaged over many rows; its tail term
is 6e-2 RMS(G) (measured worst 0.05-0.10 max|err| / RMS at RMS errors of
0.4 %, against 0.014-0.024 for the dense gradients).  Measured values are
printed.
"""
import numpy as np
import pytest
import torch

from oracle import backward as B
from tests._parity import elem_ok, make, max_rel, to64

pytestmark = pytest.mark.gpu

RMS_BAR = 1e-2
ABS_RMS = 3e-2
ROUTER_RMS_BAR = 3e-2
ROUTER_ABS_RMS = 8e-2
EXPERT_ABS_RMS = 6e-2
REL_ELEM = 2.0 ** -7


def _run(name, T=None):
    from lmoe_synth import CONFIGS, make_grad_out
    cfg = CONFIGS[name]
    w, x, layer = make(cfg, T=T, backward=True)
    T = x.shape[0]
    layer.forward(x)
    dy = make_grad_out(cfg, T=T, device="cuda")
    grads = layer.grad_buffers()
    for g in grads.values():
        g.fill_(float("nan"))          # every element must be written
    dx = layer.backward(x, dy, grads)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    S = layer.debug("topk_idx").numpy().astype(np.int64)
    ref = B.layer_backward(to64(x), to64(w["w_router"]), to64(w["router_bias"]), to64(w["w_dn"]),
                           lambda e: to64(w["w1"][e]), lambda e: to64(w["w2"][e]),
                           to64(w["w_upl"]), to64(w["w_s1"]), to64(w["w_s2"]), cfg.K, to64(dy),
                           S=S)
    return cfg, layer, grads, dx, ref, S


def _check(name, T=None):
    cfg, layer, grads, dx, ref, S = _run(name, T)
    got = {"dx": to64(dx), "dW_r": to64(grads["d_router"]), "dW_dn": to64(grads["d_dn"]),
           "dW_upl": to64(grads["d_upl"]), "dW_s1": to64(grads["d_s1"]),
           "dW_s2": to64(grads["d_s2"])}
    want = {k: ref[k] for k in got}
    # expert gradients: every expert some token chose, and zero for the rest
    gw1, gw2 = grads["d_w1"].cpu(), grads["d_w2"].cpu()
    chosen = sorted(ref["dW1"].keys())
    got["dW1"] = np.stack([gw1[e].double().numpy() for e in chosen])
    got["dW2"] = np.stack([gw2[e].double().numpy() for e in chosen])
    want["dW1"] = np.stack([ref["dW1"][e] for e in chosen])
    want["dW2"] = np.stack([ref["dW2"][e] for e in chosen])
    unused = sorted(set(range(cfg.N)) - set(chosen))
    for e in unused:
        assert not gw1[e].any() and not gw2[e].any(), f"expert {e}: no rows, nonzero gradient"
    report = {}
    for k in got:
        assert np.isfinite(got[k]).all(), f"{k}: unwritten or non-finite elements"
        rb, ab = ((ROUTER_RMS_BAR, ROUTER_ABS_RMS) if k == "dW_r" else
                  (RMS_BAR, EXPERT_ABS_RMS) if k in ("dW1", "dW2") else (RMS_BAR, ABS_RMS))
        ok, ratio, rr = elem_ok(got[k], want[k], rel=REL_ELEM, abs_rms=ab, rel_rms=rb)
        report[k] = (ok, rr, ratio, max_rel(got[k], want[k]))
    print(name, T, {k: (round(v[1], 5), round(v[2], 3), round(v[3], 4))
                    for k, v in report.items()}, "experts without rows:", len(unused))
    for k, (ok, rr, ratio, mr) in report.items():
        assert ok, f"{k}: RMS rel {rr:.3g}, elementwise error {ratio:.3g} x bound (max/RMS {mr:.3g})"
    return report


def test_backward_tiny():
    _check("tiny")


@pytest.mark.parametrize("T", [1, 50, 100])
def test_backward_tiny_ragged(T):
    """fewer rows than one 64-row box (padded staging), and a ragged tail"""
    _check("tiny", T=T)


def test_backward_multi_tile_zipf():
    """token blocks of 256 rows, several K blocks per expert segment, experts
    left without rows by the Zipf bias"""
    _check("pair_small")


def test_backward_zero_tokens_is_noop():
    from lmoe_synth import CONFIGS
    w, x, layer = make(CONFIGS["tiny"], backward=True)
    layer.forward(x[:0])
    grads = layer.grad_buffers()
    layer.backward(x[:0], x[:0], grads)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0


def test_backward_needs_flag_and_matching_T():
    from latent_space_mixture_b200 import LmoeError
    from lmoe_synth import CONFIGS
    w, x, layer = make(CONFIGS["tiny"])
    layer.forward(x)
    with pytest.raises(LmoeError):
        layer.backward(x, x, layer.grad_buffers())
    w, x, layer = make(CONFIGS["tiny"], backward=True)
    layer.forward(x)
    with pytest.raises(LmoeError):
        layer.backward(x[:10], x[:10], layer.grad_buffers())


def test_bias_update_matches_oracle():
    from lmoe_synth import CONFIGS
    cfg = CONFIGS["pair_small"]
    w, x, layer = make(cfg, backward=False)
    b0 = w["router_bias"].cpu().numpy()
    layer.forward(x)
    counts = layer.debug("counts").numpy()
    layer.bias_update(1e-3)
    torch.cuda.synchronize()
    got = layer.debug("bias").numpy()
    assert np.array_equal(got, B.bias_update(b0, counts, 1e-3))
    # the next forward routes with the updated bias
    layer.forward(x)
    counts2 = layer.debug("counts").numpy()
    assert counts2.max() <= counts.max()


def test_backward_with_an_underflowing_selected_score():
    """A selected expert whose sigmoid score underflows to 0 in float32 (its
    logit near -128, chosen through a large bias): its router weight is 0 and
    the router backward must stay finite (dz = 0 there, since s (1 - s) = 0)."""
    from lmoe_synth import CONFIGS, make_grad_out
    cfg = CONFIGS["tiny"]

    def router(t):
        t = t.clone()
        t[3] = -0.5           # z[:, 3] = -0.5 * sum(x): about -128 for x = 1
        return t

    def bias(t):
        t = t.clone()
        t[3] = 10.0           # expert 3 is always selected
        return t

    w, x, layer = make(cfg, backward=True, overrides={"w_router": router, "router_bias": bias})
    x = x.clone()
    x[:4] = 1.0
    layer.forward(x)
    dy = make_grad_out(cfg, T=x.shape[0], device="cuda")
    grads = layer.grad_buffers()
    dx = layer.backward(x, dy, grads)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    S = layer.debug("topk_idx").numpy().astype(np.int64)
    assert np.all(S[:, 0] == 3)
    assert np.all(layer.debug("topk_w").numpy()[:4, 0] == 0.0)
    ref = B.layer_backward(to64(x), to64(w["w_router"]), to64(w["router_bias"]), to64(w["w_dn"]),
                           lambda e: to64(w["w1"][e]), lambda e: to64(w["w2"][e]),
                           to64(w["w_upl"]), to64(w["w_s1"]), to64(w["w_s2"]), cfg.K, to64(dy),
                           S=S)
    for name, got in (("dx", to64(dx)), ("dW_r", to64(grads["d_router"])),
                      ("dW_dn", to64(grads["d_dn"]))):
        assert np.isfinite(got).all(), f"{name}: non-finite"
        rb, ab = (ROUTER_RMS_BAR, ROUTER_ABS_RMS) if name == "dW_r" else (RMS_BAR, ABS_RMS)
        ok, ratio, rr = elem_ok(got, ref[name], rel=REL_ELEM, abs_rms=ab, rel_rms=rb)
        assert ok, f"{name}: RMS rel {rr:.3g}, elementwise {ratio:.3g} x bound"
