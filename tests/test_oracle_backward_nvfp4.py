"""Pins of the NVFP4-recipe expert backward (oracle.backward_nvfp4): with its
quantisers and transform switched off it is the BF16 backward of the
oracle (oracle.backward, itself pinned by finite differences); the random
Hadamard transform cancels in the weight gradients (orthonormal, same signs
on both operands); stochastic rounding leaves the data gradients unbiased;
experts without rows get no gradient."""
import numpy as np

from oracle import backward as B
from oracle import backward_nvfp4 as BN


def _problem(seed, T=20, d=32, l=32, N=6, K=2, h=48, hs=16):
    rng = np.random.default_rng(seed)
    p = dict(x=rng.standard_normal((T, d)), W_r=rng.standard_normal((N, d)) * 0.3,
             b=np.zeros(N), W_dn=rng.standard_normal((l, d)) * 0.2,
             W1=rng.standard_normal((N, h, l)) * 0.2, W2=rng.standard_normal((N, l, h)) * 0.2,
             W_upl=rng.standard_normal((d, l)) * 0.2, W_s1=rng.standard_normal((hs, d)) * 0.2,
             W_s2=rng.standard_normal((d, hs)) * 0.2, G=rng.standard_normal((T, d)))
    return p, N, K


def _bf16_backward(p, K):
    return B.layer_backward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: p["W1"][e],
                            lambda e: p["W2"][e], p["W_upl"], p["W_s1"], p["W_s2"], K, p["G"])


def _nv(p, N, K, ref, **kw):
    U = p["x"] @ p["W_dn"].T
    return BN.experts_backward_nvfp4(U, ref["S"], ref["w"], ref["dv"], lambda e: p["W1"][e],
                                     lambda e: p["W2"][e], N, 0.01, 0.01, seed=11, **kw)


def test_without_quantisation_it_is_the_bf16_backward():
    p, N, K = _problem(0)
    ref = _bf16_backward(p, K)
    got = _nv(p, N, K, ref, quant_fwd=False, quant_bwd=False, rht=False)
    np.testing.assert_allclose(got["du"], ref["du"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["dw"], ref["dw"], rtol=0, atol=1e-12)
    assert sorted(got["dW1"]) == sorted(ref["dW1"])
    for e in ref["dW1"]:
        np.testing.assert_allclose(got["dW1"][e], ref["dW1"][e], rtol=0, atol=1e-12)
        np.testing.assert_allclose(got["dW2"][e], ref["dW2"][e], rtol=0, atol=1e-12)


def test_the_transform_cancels_in_the_weight_gradients():
    p, N, K = _problem(1)
    ref = _bf16_backward(p, K)
    got = _nv(p, N, K, ref, quant_fwd=False, quant_bwd=False, rht=True)
    for e in ref["dW1"]:
        s1 = np.abs(ref["dW1"][e]).max()
        np.testing.assert_allclose(got["dW1"][e], ref["dW1"][e], rtol=0, atol=1e-5 * s1)
        s2 = np.abs(ref["dW2"][e]).max()
        np.testing.assert_allclose(got["dW2"][e], ref["dW2"][e], rtol=0, atol=1e-5 * s2)


def test_stochastic_rounding_leaves_the_data_gradient_unbiased():
    """Averaged over seeds, du with quantised gradients approaches du of the
    same (quantised) forward with unquantised gradients."""
    p, N, K = _problem(2)
    ref = _bf16_backward(p, K)
    U = p["x"] @ p["W_dn"].T
    exact = BN.experts_backward_nvfp4(U, ref["S"], ref["w"], ref["dv"], lambda e: p["W1"][e],
                                      lambda e: p["W2"][e], N, 0.01, 0.01, seed=0,
                                      quant_fwd=True, quant_bwd=False)["du"]
    n = 300
    acc = np.zeros_like(exact)
    one = None
    for s in range(n):
        du = BN.experts_backward_nvfp4(U, ref["S"], ref["w"], ref["dv"], lambda e: p["W1"][e],
                                       lambda e: p["W2"][e], N, 0.01, 0.01, seed=100 * s,
                                       quant_fwd=True, quant_bwd=True)["du"]
        acc += du
        one = du if one is None else one
    rms = np.sqrt(np.mean(exact ** 2))
    err_one = np.sqrt(np.mean((one - exact) ** 2)) / rms
    err_mean = np.sqrt(np.mean((acc / n - exact) ** 2)) / rms
    assert err_one > 0.02                      # one draw carries the rounding noise
    assert err_mean < 3.0 * err_one / np.sqrt(n)   # the mean converges as 1/sqrt(n)


def test_experts_without_rows_get_no_gradient_and_shapes():
    p, N, K = _problem(3, N=8, K=1, T=5)
    ref = _bf16_backward(p, K)
    got = _nv(p, N, K, ref)
    used = set(np.unique(ref["S"]).tolist())
    assert set(got["dW1"]) == used and set(got["dW2"]) == used
    for e in used:
        assert got["dW1"][e].shape == (48, 32) and got["dW2"][e].shape == (32, 48)
    assert got["du"].shape == (5, 32) and np.isfinite(got["du"]).all()
