"""Pins of the oracle's backward pass and of its aux-loss-free bias update.

The backward is pinned against central finite differences of the oracle's
own forward (a different program: it only evaluates the layer), against
torch autograd of the forward restated in torch (a library routine doing the
differentiation), and against closed forms: K = 1 (w = 1 whatever the router
says, so the router weight gets no gradient), W1 = 0 (no expert gradient
reaches W_dn or W_upl) and the standard MoE (no projections).
"""
import numpy as np
import pytest
import torch

from oracle import backward as B
from oracle import lmoe as O


def _problem(seed, T=3, d=8, l=4, N=5, K=2, h=3, hs=4, latent=True, scale=0.5):
    rng = np.random.default_rng(seed)
    p = dict(x=rng.standard_normal((T, d)),
             W_r=rng.standard_normal((N, d)) * scale,
             b=rng.standard_normal(N) * 0.1,
             W_dn=rng.standard_normal((l if latent else d, d)) * scale if latent else None,
             W1=rng.standard_normal((N, h, l if latent else d)) * scale,
             W2=rng.standard_normal((N, l if latent else d, h)) * scale,
             W_upl=rng.standard_normal((d, l)) * scale if latent else None,
             W_s1=rng.standard_normal((hs, d)) * scale,
             W_s2=rng.standard_normal((d, hs)) * scale,
             G=rng.standard_normal((T, d)), K=K)
    return p


def _fwd(p, **over):
    q = dict(p, **over)
    return O.layer_forward(q["x"], q["W_r"], q["b"], q["W_dn"], lambda e: q["W1"][e],
                           lambda e: q["W2"][e], q["W_upl"], q["W_s1"], q["W_s2"], q["K"])


def _bwd(p):
    return B.layer_backward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: p["W1"][e],
                            lambda e: p["W2"][e], p["W_upl"], p["W_s1"], p["W_s2"], p["K"],
                            p["G"])


def _dense(g, name, p):
    """dW1 / dW2 dicts -> full [N][...] arrays (zeros for unselected experts)."""
    full = np.zeros_like(p[name])
    for e, v in g.items():
        full[e] = v
    return full


def _loss(p, **over):
    return float(np.sum(_fwd(p, **over)["y"] * p["G"]))


def _fd_check(p, name, grad, eps=1e-6, rtol=1e-6):
    base_S = _fwd(p)["S"]
    arr = p[name]
    num = np.zeros_like(arr)
    for idx in np.ndindex(arr.shape):
        plus, minus = arr.copy(), arr.copy()
        plus[idx] += eps
        minus[idx] -= eps
        # the selection must not change under the probe (it is piecewise constant)
        assert np.array_equal(_fwd(p, **{name: plus})["S"], base_S)
        assert np.array_equal(_fwd(p, **{name: minus})["S"], base_S)
        num[idx] = (_loss(p, **{name: plus}) - _loss(p, **{name: minus})) / (2 * eps)
    scale = max(np.abs(num).max(), 1e-12)
    assert np.abs(grad - num).max() <= rtol * scale + 1e-9, name


@pytest.mark.parametrize("seed", [0, 1])
def test_backward_matches_finite_differences(seed):
    p = _problem(seed)
    assert _fwd(p)["gap"].min() > 1e-3   # probes of 1e-6 cannot flip the selection
    g = _bwd(p)
    _fd_check(p, "x", g["dx"])
    _fd_check(p, "W_r", g["dW_r"])
    _fd_check(p, "W_dn", g["dW_dn"])
    _fd_check(p, "W1", _dense(g["dW1"], "W1", p))
    _fd_check(p, "W2", _dense(g["dW2"], "W2", p))
    _fd_check(p, "W_upl", g["dW_upl"])
    _fd_check(p, "W_s1", g["dW_s1"])
    _fd_check(p, "W_s2", g["dW_s2"])


def test_backward_standard_moe_matches_finite_differences():
    p = _problem(4, latent=False, d=6)
    g = _bwd(p)
    assert g["dW_dn"] is None and g["dW_upl"] is None
    _fd_check(p, "x", g["dx"])
    _fd_check(p, "W1", _dense(g["dW1"], "W1", p))
    _fd_check(p, "W2", _dense(g["dW2"], "W2", p))
    _fd_check(p, "W_r", g["dW_r"])


def test_backward_matches_torch_autograd():
    """The forward restated in torch with the selection held fixed, then
    torch.autograd differentiates it."""
    p = _problem(7, T=6, d=16, l=8, N=7, K=3, h=5, hs=6)
    g = _bwd(p)
    S = torch.from_numpy(g["S"])
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True)
         for k, v in p.items() if isinstance(v, np.ndarray) and k not in ("b", "G")}
    s = torch.sigmoid(t["x"] @ t["W_r"].T)
    ssel = torch.gather(s, 1, S)
    w = ssel / ssel.sum(1, keepdim=True)
    u = t["x"] @ t["W_dn"].T
    v = torch.zeros_like(u)
    for ti in range(S.shape[0]):
        for k in range(S.shape[1]):
            e = int(S[ti, k])
            a = t["W1"][e] @ u[ti]
            v = v.index_add(0, torch.tensor([ti]),
                            (w[ti, k] * (t["W2"][e] @ torch.relu(a) ** 2))[None])
    y = v @ t["W_upl"].T + torch.relu(t["x"] @ t["W_s1"].T) ** 2 @ t["W_s2"].T
    (y * torch.from_numpy(p["G"])).sum().backward()
    ref = {"dx": t["x"].grad, "dW_r": t["W_r"].grad, "dW_dn": t["W_dn"].grad,
           "dW_upl": t["W_upl"].grad, "dW_s1": t["W_s1"].grad, "dW_s2": t["W_s2"].grad}
    for k, r in ref.items():
        np.testing.assert_allclose(g[k], r.numpy(), rtol=1e-10, atol=1e-12, err_msg=k)
    np.testing.assert_allclose(_dense(g["dW1"], "W1", p), t["W1"].grad.numpy(), rtol=1e-10,
                               atol=1e-12)
    np.testing.assert_allclose(_dense(g["dW2"], "W2", p), t["W2"].grad.numpy(), rtol=1e-10,
                               atol=1e-12)


def test_top1_router_gets_no_gradient():
    """K = 1: w = s / s = 1 for every router output, so dL/dW_r = 0 exactly
    and the layer is a dense FFN per token."""
    p = _problem(2, K=1)
    g = _bwd(p)
    assert np.array_equal(g["dW_r"], np.zeros_like(p["W_r"]))
    assert np.array_equal(g["w"], np.ones_like(g["w"]))


def test_zero_expert_weights_cut_the_routed_gradient():
    """W1 = 0: the experts output 0 whatever u is, so no gradient reaches
    W_dn, W_upl, W2 or the router; dx is the shared expert's alone."""
    p = _problem(3)
    p["W1"] = np.zeros_like(p["W1"])
    g = _bwd(p)
    for k in ("dW_dn", "dW_upl", "dW_r"):
        assert np.array_equal(g[k], np.zeros_like(g[k])), k
    assert all(not v.any() for v in g["dW2"].values())
    shared_only = (p["G"] @ p["W_s2"] * 2 * np.maximum(p["x"] @ p["W_s1"].T, 0)) @ p["W_s1"]
    np.testing.assert_allclose(g["dx"], shared_only, rtol=1e-12, atol=1e-14)


def test_router_gradient_sums_to_zero_over_the_selection():
    """sum_k ds_k s_k = 0: scaling every selected score by one factor leaves w
    unchanged, so the gradient has no component along s_S."""
    p = _problem(5, T=4, d=12, N=9, K=4)
    g = _bwd(p)
    s = O.sigmoid(p["x"] @ p["W_r"].T)
    ssel = np.take_along_axis(s, g["S"], axis=1)
    ds = np.take_along_axis(g["dz"], g["S"], axis=1) / (ssel * (1 - ssel))
    np.testing.assert_allclose(np.sum(ds * ssel, axis=1), 0.0, atol=1e-12)


def test_bias_update_rule():
    b = np.zeros(4, dtype=np.float32)
    # T*K = 8 rows over 4 experts: mean 2
    nb = B.bias_update(b, np.array([5, 2, 1, 0]))
    assert nb.dtype == np.float32
    r = np.float32(1e-3)
    assert np.array_equal(nb, np.array([-r, 0, r, r], dtype=np.float32))
    # balanced load leaves the bias where it is
    b2 = np.array([0.5, -0.25, 0.125], dtype=np.float32)
    assert np.array_equal(B.bias_update(b2, np.array([3, 3, 3])), b2)
    # a mean that is not an integer: 7 rows over 2 experts
    assert np.array_equal(B.bias_update(np.zeros(2, np.float32), np.array([4, 3])),
                          np.array([-r, r], dtype=np.float32))
    assert B.BIAS_UPDATE_RATE == 1e-3


def test_bias_update_moves_selection_toward_balance():
    """Repeated updates on a fixed batch shrink the max/mean load (the point
    of the rule), starting from a Zipf-skewed bias."""
    rng = np.random.default_rng(11)
    T, d, N, K = 256, 16, 16, 2
    x = rng.standard_normal((T, d))
    W_r = rng.standard_normal((N, d)) * 0.3
    b = (0.1 * np.log((1.0 + rng.permutation(N)) ** -1.1)).astype(np.float32)
    def load(bias):
        S, _, _, _ = O.route(x @ W_r.T, bias.astype(np.float64), K)
        return np.bincount(S.reshape(-1), minlength=N)
    c0 = load(b)
    for _ in range(300):
        b = B.bias_update(b, load(b), rate=2e-3)
    c1 = load(b)
    assert c1.max() < c0.max()
    assert c1.max() / c1.mean() < 1.6
