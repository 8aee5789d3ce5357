"""Pins of the oracle's NVFP4 gradient-path pieces (oracle.nvfp4_train):
the counter-based generator against its published first outputs, the random
Hadamard transform against scipy's Hadamard matrix (a library routine) and
its orthonormality, and stochastic rounding against its defining property
(unbiased in expectation) and its special cases."""
import numpy as np
import scipy.linalg

from oracle import nvfp4 as Q
from oracle import nvfp4_train as T


def test_splitmix64_first_outputs():
    """SplitMix64 with seed 0: the sequence its authors' reference code prints."""
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F,
            0xF88BB8A8724C81EC, 0x1B39896A51A8749B]
    got = T.splitmix64(0, np.arange(5, dtype=np.uint64))
    assert [int(v) for v in got] == want


def test_uniform24_is_uniform_and_in_range():
    u = T.uniform24(12345, np.arange(1 << 20, dtype=np.uint64)).astype(np.float64)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 2e-3
    assert abs(u.var() - 1.0 / 12.0) < 1e-3
    # 24-bit grid
    assert np.all(np.round(u * 2 ** 24) == u * 2 ** 24)


def test_rht16_is_the_scaled_hadamard_matrix():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((5, 64)).astype(np.float32)
    H = scipy.linalg.hadamard(16).astype(np.float64) / 4.0
    ones = np.ones(16, dtype=np.float32)
    got = T.rht16(X, signs=ones).astype(np.float64)
    want = (X.astype(np.float64).reshape(-1, 16) @ H.T).reshape(X.shape)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-5)
    s = T.rht_signs(7)
    assert set(np.unique(s).tolist()) <= {-1.0, 1.0} and (s < 0).any() and (s > 0).any()
    got = T.rht16(X, seed=7).astype(np.float64)
    want = ((X.astype(np.float64).reshape(-1, 16) * s) @ H.T).reshape(X.shape)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-5)


def test_rht16_is_orthonormal_and_inverted_by_itself():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((8, 32)).astype(np.float32)
    Y = T.rht16(X, seed=3)
    nb = lambda A: np.linalg.norm(A.astype(np.float64).reshape(-1, 16), axis=1)  # noqa: E731
    np.testing.assert_allclose(nb(Y), nb(X), rtol=1e-6)
    back = T.rht16(Y, signs=np.ones(16, np.float32)) * T.rht_signs(3)[None, :].repeat(2, 0).reshape(-1)
    np.testing.assert_allclose(back, X, rtol=0, atol=1e-5)


def test_rht16_exact_on_a_single_spike():
    """A block with one nonzero element x_j becomes +-x_j / 4 everywhere."""
    X = np.zeros((1, 16), np.float32)
    X[0, 5] = 3.0
    Y = T.rht16(X, signs=np.ones(16, np.float32))
    assert np.array_equal(np.abs(Y), np.full((1, 16), 0.75, np.float32))


def test_sr_special_cases():
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.5, -6.0, 7.5, -100.0], np.float32)
    for u in (0.0, 0.5, 0.999):
        codes = T.e2m1_sr(grid, np.full(grid.shape, u, np.float32))
        assert np.array_equal(Q.e2m1_decode(codes), np.clip(grid, -6, 6).astype(np.float64))
    # between 1.5 and 2 at a quarter of the way: up when u < 0.25
    v = np.full(4, 1.625, np.float32)
    codes = T.e2m1_sr(v, np.array([0.0, 0.2499, 0.25, 0.9], np.float32))
    assert np.array_equal(Q.e2m1_decode(codes), [2.0, 2.0, 1.5, 1.5])
    # the sign follows the value, including -0
    c = T.e2m1_sr(np.array([-0.0, -0.2], np.float32), np.array([0.9, 0.9], np.float32))
    assert np.array_equal(c, [8, 8])


def test_sr_is_unbiased_in_expectation():
    """E[SR(v)] = v: the mean over many independent draws converges to v."""
    rng = np.random.default_rng(2)
    v = rng.uniform(-6, 6, 64).astype(np.float32)
    n = 20000
    u = T.uniform24(99, np.arange(64 * n, dtype=np.uint64)).reshape(n, 64)
    mean = Q.e2m1_decode(T.e2m1_sr(np.broadcast_to(v, (n, 64)), u)).mean(axis=0)
    # per element std <= half a grid step (1) / sqrt(n)
    assert np.max(np.abs(mean - v)) < 5.0 / np.sqrt(n)
    # round-to-nearest is biased on the same values
    rn = Q.e2m1_decode(Q.e2m1_rtne(v))
    assert np.max(np.abs(rn - v)) > 0.1


def test_quantize_sr_keeps_the_round_to_nearest_scales():
    rng = np.random.default_rng(3)
    X = (rng.standard_normal((6, 48)) * np.exp(rng.uniform(-3, 3, (6, 1)))).astype(np.float32)
    X[2, 16:32] = 0.0
    g = np.float32(0.01)
    codes, sc, sb = T.quantize_sr(X, g, seed=5)
    _, sc_rn, _ = Q.quantize(X, g)
    assert np.array_equal(sc, sc_rn)
    # every element rounds to one of the two neighbours of its scaled value
    deq = T.fake_quant_sr(X, g, seed=5)
    rn = Q.fake_quant(X, g)
    step = np.repeat(sb.astype(np.float64), 16, axis=1) * np.float64(g) * 2.0
    assert np.all(np.abs(deq - X) <= step + 1e-12)
    assert not np.array_equal(deq, rn)   # some elements went the other way
    assert np.all(codes[2, 16:32] & 7 == 0)
    # different seeds give different roundings, the same seed the same
    assert np.array_equal(T.quantize_sr(X, g, seed=5)[0], codes)
    assert not np.array_equal(T.quantize_sr(X, g, seed=6)[0], codes)
