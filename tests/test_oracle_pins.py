"""Pins of the float64 oracle to things other than itself.

Each test ties an oracle function to the pages (golden fixtures), to a closed
form, to an invariant, or to a brute-force restatement written with plain
loops, so that a plausible mistake in the oracle (a dropped term, a wrong
sign, a transposed operand, bias in the weights, no renormalisation, a wrong
tie-break) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from oracle import lmoe as O


# ----------------------------------------------------------------------------
# helpers: loop-only restatement (no numpy linear algebra)


def _matvec(W, x):
    return [sum(W[i][j] * x[j] for j in range(len(x))) for i in range(len(W))]


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def _dense_masked_layer(x, W_r, b, W_dn, W1, W2, W_upl, W_s1, W_s2, K):
    """Every expert on every token, times a 0/1 mask and the weight.

    The mask comes from brute force over all K-subsets (the subset with the
    largest sum of keys), not from sorting.
    """
    T, N = len(x), len(W_r)
    ys = []
    for t in range(T):
        z = _matvec(W_r, x[t])
        s = [_sig(v) for v in z]
        key = [s[e] + b[e] for e in range(N)]
        best = max(itertools.combinations(range(N), K),
                   key=lambda c: sum(key[e] for e in c))
        mask = [1.0 if e in best else 0.0 for e in range(N)]
        denom = sum(s[e] * mask[e] for e in range(N))
        u = _matvec(W_dn, x[t])
        v = [0.0] * len(u)
        for e in range(N):
            a = _matvec(W1[e], u)
            g = [max(ai, 0.0) ** 2 for ai in a]
            o = _matvec(W2[e], g)
            for i in range(len(v)):
                v[i] += mask[e] * (s[e] / denom) * o[i]
        r = _matvec(W_upl, v)
        hs = [max(a, 0.0) ** 2 for a in _matvec(W_s1, x[t])]
        sh = _matvec(W_s2, hs)
        ys.append([r[i] + sh[i] for i in range(len(r))])
    return np.array(ys)


def _rand_layer(rng, T, d, l, N, h, hs, bias_scale=0.0):
    return dict(
        x=rng.standard_normal((T, d)),
        W_r=rng.standard_normal((N, d)) * 0.5,
        b=rng.standard_normal(N) * bias_scale,
        W_dn=rng.standard_normal((l, d)) * 0.5,
        W1=rng.standard_normal((N, h, l)) * 0.5,
        W2=rng.standard_normal((N, l, h)) * 0.5,
        W_upl=rng.standard_normal((d, l)) * 0.5,
        W_s1=rng.standard_normal((hs, d)) * 0.5,
        W_s2=rng.standard_normal((d, hs)) * 0.5,
    )


def _oracle(p, K, quant=None):
    return O.layer_forward(p["x"], p["W_r"], p["b"], p["W_dn"],
                           lambda e: p["W1"][e], lambda e: p["W2"][e],
                           p["W_upl"], p["W_s1"], p["W_s2"], K, quant=quant)


# ----------------------------------------------------------------------------
# routing


@pytest.mark.parametrize("N,K", [(5, 2), (7, 3), (10, 4), (6, 1), (8, 8)])
def test_topk_matches_brute_force_subsets(N, K):
    rng = np.random.default_rng(100 + N * 10 + K)
    z = rng.standard_normal((20, N))
    b = rng.standard_normal(N) * 0.3
    S, w, gap, s = O.route(z, b, K)
    key = 1.0 / (1.0 + np.exp(-z)) + b
    for t in range(20):
        best = max(itertools.combinations(range(N), K),
                   key=lambda c: sum(key[t, e] for e in c))
        assert set(S[t].tolist()) == set(best)
        # slot order: key descending
        ks = key[t, S[t]]
        assert np.all(np.diff(ks) <= 0)


def test_weights_sum_to_one_and_use_unbiased_scores():
    rng = np.random.default_rng(1)
    z = rng.standard_normal((50, 16))
    b = rng.standard_normal(16)
    S, w, gap, s = O.route(z, b, 4)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-15, rtol=0)
    sig = 1.0 / (1.0 + np.exp(-z))
    for t in range(50):
        sel = sig[t, S[t]]
        assert np.allclose(w[t], sel / sel.sum(), atol=1e-15, rtol=0)


def test_bias_changes_selection_but_not_weights_closed_form():
    # z = [0, ln 3, -ln 3]: s = [1/2, 3/4, 1/4].  Without bias the top-2 is
    # {1, 0} with w = [0.6, 0.4].  With b = [0, 0, 0.6] the keys are
    # [0.5, 0.75, 0.85]: top-2 is [2, 1] and w = [1/4, 3/4] / 1 = [0.25, 0.75].
    z = np.array([[0.0, math.log(3.0), -math.log(3.0)]])
    S, w, _, _ = O.route(z, None, 2)
    assert S[0].tolist() == [1, 0]
    assert np.allclose(w[0], [0.6, 0.4], atol=1e-15)
    S, w, _, _ = O.route(z, np.array([0.0, 0.0, 0.6]), 2)
    assert S[0].tolist() == [2, 1]
    assert np.allclose(w[0], [0.25, 0.75], atol=1e-15)


def test_ties_go_to_lower_expert_id():
    z = np.zeros((1, 6))                         # all scores exactly 1/2
    S, w, gap, _ = O.route(z, None, 3)
    assert S[0].tolist() == [0, 1, 2]
    assert gap[0] == 0.0
    assert np.allclose(w[0], [1 / 3] * 3, atol=1e-15)
    z = np.array([[0.0, 1.0, 1.0, 0.0, 1.0]])
    S, _, _, _ = O.route(z, None, 2)
    assert S[0].tolist() == [1, 2]


def test_k_equals_n_selects_all():
    rng = np.random.default_rng(5)
    z = rng.standard_normal((4, 7))
    S, w, gap, _ = O.route(z, None, 7)
    sig = 1.0 / (1.0 + np.exp(-z))
    for t in range(4):
        assert sorted(S[t].tolist()) == list(range(7))
        assert np.allclose(w[t], sig[t, S[t]] / sig[t].sum(), atol=1e-15)
    assert np.all(np.isinf(gap))


def test_sigmoid_closed_forms():
    assert O.sigmoid(0.0) == 0.5
    assert abs(O.sigmoid(math.log(3.0)) - 0.75) < 1e-15
    assert abs(O.sigmoid(-math.log(3.0)) - 0.25) < 1e-15
    assert abs(O.sigmoid(-40.0) - math.exp(-40.0)) < 1e-30


def test_gap_is_kth_minus_next():
    z = np.array([[2.0, -1.0, 0.5, 0.0]])
    S, _, gap, _ = O.route(z, None, 2)
    assert S[0].tolist() == [0, 2]
    assert abs(gap[0] - (_sig(0.5) - _sig(0.0))) < 1e-15


def test_is_valid_topk():
    key = np.array([0.9, 0.5, 0.5004, 0.1])
    assert O.is_valid_topk(key, [0, 2], 0.0)
    assert not O.is_valid_topk(key, [0, 1], 0.0)
    assert O.is_valid_topk(key, [0, 1], 1e-3)
    assert not O.is_valid_topk(key, [0, 3], 1e-3)
    assert not O.is_valid_topk(key, [0, 0], 1.0)


# ----------------------------------------------------------------------------
# segments (per-expert rows)


def _brute_segments(S, N):
    T, K = S.shape
    entries = sorted((int(S[t, k]), t, k) for t in range(T) for k in range(K))
    perm = [t * K + k for (_, t, k) in entries]
    counts = [sum(1 for (e, _, _) in entries if e == x) for x in range(N)]
    return counts, perm


@pytest.mark.parametrize("T,N,K", [(13, 8, 3), (40, 32, 4), (1, 5, 5), (64, 16, 1)])
def test_segments_equal_stable_sort_and_invert(T, N, K):
    rng = np.random.default_rng(T * N + K)
    S = np.stack([rng.permutation(N)[:K] for _ in range(T)])
    counts, offsets, perm, inv = O.segments(S, N)
    c2, p2 = _brute_segments(S, N)
    assert counts.tolist() == c2
    assert perm.tolist() == p2
    assert counts.sum() == T * K
    assert offsets[0] == 0 and offsets[-1] == T * K
    assert np.all(np.diff(offsets) == counts)
    # perm o inv = identity, and gather then scatter returns the input
    for t in range(T):
        for k in range(K):
            assert perm[inv[t, k]] == t * K + k
    data = rng.standard_normal((T, K, 3))
    gathered = data.reshape(T * K, 3)[perm]
    back = np.empty_like(data)
    back[np.arange(T)[:, None], np.arange(K)[None, :]] = gathered[inv]
    assert np.array_equal(back, data)
    # rows of expert e hold ascending tokens
    for e in range(N):
        rows = perm[offsets[e]:offsets[e + 1]] // K
        assert np.all(np.diff(rows) > 0)
        assert np.all(S.reshape(-1)[perm[offsets[e]:offsets[e + 1]]] == e)


def test_segments_empty_experts():
    S = np.array([[3, 1], [1, 3], [3, 0]])
    counts, offsets, perm, inv = O.segments(S, 6)
    assert counts.tolist() == [1, 2, 0, 3, 0, 0]
    assert offsets.tolist() == [0, 1, 3, 3, 6, 6, 6]
    # expert 0: (t2, k1) -> 5; expert 1: (t0, k1) -> 1, (t1, k0) -> 2;
    # expert 3: (t0, k0) -> 0, (t1, k1) -> 3, (t2, k0) -> 4
    assert perm.tolist() == [5, 1, 2, 0, 3, 4]
    assert inv.tolist() == [[3, 1], [2, 4], [5, 0]]


# ----------------------------------------------------------------------------
# the layer: hand-worked example, loop-only restatement, special cases


def test_hand_worked_tiny_layer():
    """T=1, d=2, l=2, N=3, K=2, h=2, h_s=2, computed by hand.

    x = [1, 1]; z = W_r x = [0, ln3, -ln3] -> s = [1/2, 3/4, 1/4]
    top-2 = [1, 0], w = [0.75, 0.5] / 1.25 = [0.6, 0.4]
    u = W_dn x = [[1,0],[1,1]] [1,1] = [1, 2]
    expert 1: a = [[1,1],[0,1]] u = [3, 2] -> g = [9, 4]
              o1 = [[1,0],[1,-1]] g = [9, 5]
    expert 0: a = [[2,-2],[1,1]] u = [-2, 3] -> g = [0, 9]
              o0 = [[0,1],[0,2]] g = [9, 18]
    v = 0.6 [9, 5] + 0.4 [9, 18] = [9.0, 10.2]
    r = [[1,0],[1,-1]] v = [9.0, -1.2]
    shared: [[3,0],[-1,-1]] x = [3, -2] -> [9, 0]; [[1,2],[-1,1]] [9,0] = [9, -9]
    y = [18.0, -10.2]
    """
    L3 = math.log(3.0)
    p = dict(
        x=np.array([[1.0, 1.0]]),
        W_r=np.array([[0.0, 0.0], [L3, 0.0], [-L3, 0.0]]),
        b=np.zeros(3),
        W_dn=np.array([[1.0, 0.0], [1.0, 1.0]]),
        W1=np.array([[[2.0, -2.0], [1.0, 1.0]],
                     [[1.0, 1.0], [0.0, 1.0]],
                     [[5.0, 5.0], [5.0, 5.0]]]),
        W2=np.array([[[0.0, 1.0], [0.0, 2.0]],
                     [[1.0, 0.0], [1.0, -1.0]],
                     [[1.0, 1.0], [1.0, 1.0]]]),
        W_upl=np.array([[1.0, 0.0], [1.0, -1.0]]),
        W_s1=np.array([[3.0, 0.0], [-1.0, -1.0]]),
        W_s2=np.array([[1.0, 2.0], [-1.0, 1.0]]),
    )
    out = _oracle(p, 2)
    assert out["S"][0].tolist() == [1, 0]
    assert np.allclose(out["w"][0], [0.6, 0.4], atol=1e-14)
    assert np.allclose(out["u"][0], [1.0, 2.0], atol=0)
    assert np.allclose(out["v"][0], [9.0, 10.2], atol=1e-13)
    assert np.allclose(out["r"][0], [9.0, -1.2], atol=1e-13)
    assert np.allclose(out["sh"][0], [9.0, -9.0], atol=0)
    assert np.allclose(out["y"][0], [18.0, -10.2], atol=1e-13)


@pytest.mark.parametrize("seed,bias_scale", [(0, 0.0), (1, 0.4), (2, 0.0)])
def test_layer_matches_loop_only_dense_masked_restatement(seed, bias_scale):
    rng = np.random.default_rng(seed)
    T, d, l, N, K, h, hs = 3, 8, 4, 5, 2, 3, 4
    p = _rand_layer(rng, T, d, l, N, h, hs, bias_scale)
    y_ref = _dense_masked_layer(p["x"].tolist(), p["W_r"].tolist(), p["b"].tolist(),
                                p["W_dn"].tolist(), p["W1"].tolist(), p["W2"].tolist(),
                                p["W_upl"].tolist(), p["W_s1"].tolist(),
                                p["W_s2"].tolist(), K)
    out = _oracle(p, K)
    assert np.allclose(out["y"], y_ref, atol=1e-12, rtol=0)


def test_single_expert_reduces_to_dense_ffn():
    rng = np.random.default_rng(7)
    T, d, l, h, hs = 5, 12, 6, 7, 9
    p = _rand_layer(rng, T, d, l, 1, h, hs)
    out = _oracle(p, 1)
    assert np.all(out["w"] == 1.0)
    x = p["x"]
    u = x @ p["W_dn"].T
    dense = np.maximum(u @ p["W1"][0].T, 0) ** 2 @ p["W2"][0].T @ p["W_upl"].T
    shared = np.maximum(x @ p["W_s1"].T, 0) ** 2 @ p["W_s2"].T
    assert np.allclose(out["y"], dense + shared, atol=1e-12, rtol=0)


def test_identity_projections_give_standard_moe():
    """l = d and W_dn = W_upl = I: a standard (non-latent) MoE layer."""
    rng = np.random.default_rng(8)
    T, d, N, K, h, hs = 6, 5, 4, 2, 3, 4
    p = _rand_layer(rng, T, d, d, N, h, hs)
    p["W_dn"] = np.eye(d)
    p["W_upl"] = np.eye(d)
    out = _oracle(p, K)
    x = p["x"]
    sig = 1.0 / (1.0 + np.exp(-(x @ p["W_r"].T)))
    y = np.maximum(x @ p["W_s1"].T, 0) ** 2 @ p["W_s2"].T
    for t in range(T):
        top = np.argsort(-sig[t], kind="stable")[:K]
        ws = sig[t, top] / sig[t, top].sum()
        for wk, e in zip(ws, top):
            y[t] += wk * (p["W2"][e] @ np.maximum(p["W1"][e] @ x[t], 0) ** 2)
    assert np.allclose(out["y"], y, atol=1e-12, rtol=0)


@pytest.mark.parametrize("seed,bias_scale", [(3, 0.0), (4, 0.4)])
def test_standard_moe_matches_loop_only_restatement(seed, bias_scale):
    """No projections (W_dn = W_upl = None): the loop restatement with u = x
    and r = v, every expert on every token under a brute-force mask."""
    rng = np.random.default_rng(seed)
    T, d, N, K, h, hs = 3, 6, 5, 2, 3, 4
    p = _rand_layer(rng, T, d, d, N, h, hs, bias_scale)
    eye = np.eye(d).tolist()
    y_ref = _dense_masked_layer(p["x"].tolist(), p["W_r"].tolist(), p["b"].tolist(), eye,
                                p["W1"].tolist(), p["W2"].tolist(), eye,
                                p["W_s1"].tolist(), p["W_s2"].tolist(), K)
    p["W_dn"] = None
    p["W_upl"] = None
    out = _oracle(p, K)
    assert np.allclose(out["y"], y_ref, atol=1e-12, rtol=0)
    assert np.array_equal(out["u"], p["x"])
    assert np.array_equal(out["r"], out["v"])


def test_standard_moe_equals_identity_projections_exactly():
    rng = np.random.default_rng(12)
    T, d, N, K, h, hs = 7, 8, 6, 3, 5, 4
    p = _rand_layer(rng, T, d, d, N, h, hs, 0.3)
    q = dict(p, W_dn=np.eye(d), W_upl=np.eye(d))
    p["W_dn"] = None
    p["W_upl"] = None
    a, b = _oracle(p, K), _oracle(q, K)
    for k in ("S", "w", "u", "v", "r", "sh", "y"):
        assert np.array_equal(a[k], b[k]), k
    t = 2
    tf = O.token_forward(p["x"][t], a["S"][t], a["s"][t], None, lambda e: p["W1"][e],
                         lambda e: p["W2"][e], None)
    assert np.allclose(tf["r"], a["r"][t], atol=1e-14, rtol=0)
    with pytest.raises(ValueError):
        O.layer_forward(p["x"], p["W_r"], p["b"], np.eye(d), lambda e: p["W1"][e],
                        lambda e: p["W2"][e], None, p["W_s1"], p["W_s2"], K)


def test_zero_w1_gives_shared_only():
    rng = np.random.default_rng(9)
    p = _rand_layer(rng, 4, 8, 4, 6, 3, 5)
    p["W1"] = np.zeros_like(p["W1"])
    out = _oracle(p, 3)
    assert np.all(out["r"] == 0.0)
    assert np.array_equal(out["y"], out["sh"])


def test_latent_combine_equals_per_expert_projection():
    """sum_k w_k W_upl o_k = W_upl (sum_k w_k o_k): combining in latent space
    before the one up-projection is exact (linearity of W_upl)."""
    rng = np.random.default_rng(10)
    T, d, l, N, K, h, hs = 4, 10, 3, 6, 3, 5, 4
    p = _rand_layer(rng, T, d, l, N, h, hs)
    out = _oracle(p, K)
    u = p["x"] @ p["W_dn"].T
    r = np.zeros((T, d))
    for t in range(T):
        for k in range(K):
            e = out["S"][t, k]
            o = p["W2"][e] @ np.maximum(p["W1"][e] @ u[t], 0) ** 2
            r[t] += out["w"][t, k] * (p["W_upl"] @ o)
    assert np.allclose(out["r"], r, atol=1e-12, rtol=0)


def test_tokens_are_independent():
    rng = np.random.default_rng(11)
    p = _rand_layer(rng, 9, 8, 4, 6, 3, 5, bias_scale=0.2)
    full = _oracle(p, 2)
    idx = [7, 2, 5]
    q = dict(p, x=p["x"][idx])
    sub = _oracle(q, 2)
    assert np.array_equal(sub["S"], full["S"][idx])
    assert np.allclose(sub["y"], full["y"][idx], atol=1e-13, rtol=0)


def test_token_forward_matches_layer_for_its_own_set():
    rng = np.random.default_rng(12)
    p = _rand_layer(rng, 5, 8, 4, 6, 3, 5)
    out = _oracle(p, 3)
    for t in range(5):
        tf = O.token_forward(p["x"][t], out["S"][t], out["s"][t], p["W_dn"],
                             lambda e: p["W1"][e], lambda e: p["W2"][e], p["W_upl"])
        assert np.allclose(tf["v"], out["v"][t], atol=1e-13)
        assert np.allclose(tf["r"], out["r"][t], atol=1e-13)


# ----------------------------------------------------------------------------
# eq.(1) and the pages' layer tables


def test_scaling_relation_eq1(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "eq1_scaling.json")))
    Np, Kp = O.scaling_relation(g["N"], g["K"], g["d"], g["l"])
    assert Np == g["N_prime_printed"] == 512
    assert Kp == 24                        # eq.(1) exactly
    assert g["K_prime_printed"] == 22 <= Kp  # the published choice
    with pytest.raises(ValueError):
        O.scaling_relation(5, 3, 10, 4)


def test_workload_dims_follow_the_pages_tables(golden_dir):
    from lmoe_synth import CONFIGS
    g = json.load(open(os.path.join(golden_dir, "layer_dims.json")))
    for name in ("super_decode", "super_prefill", "super_prefill_nvfp4"):
        c = CONFIGS[name]
        s = g["super"]
        assert (c.d, c.h, c.hs, c.N, c.K, c.l) == (
            s["d"], s["expert_hidden"], s["shared_hidden"], s["n_experts"],
            s["top_k"], s["latent"])
    c, u = CONFIGS["ultra"], g["ultra"]
    assert (c.d, c.h, c.hs, c.N, c.K, c.l) == (
        u["d"], u["expert_hidden"], u["shared_hidden"], u["n_experts"],
        u["top_k"], u["latent"])
    # the Super layer is eq.(1) applied to a 128-expert top-6 layer at d/l = 4
    s = g["super"]
    assert O.scaling_relation(128, 6, s["d"], s["latent"])[0] == s["n_experts"]
    # the standard-MoE comparator: the pages' 128 experts, top 6, at width d,
    # with Super's expert widths: expert parameters N h l match in total
    m = g["standard_moe"]
    for name in ("std_decode", "std_prefill"):
        c = CONFIGS[name]
        assert not c.proj and c.l == c.d == m["d"]
        assert (c.N, c.K) == (m["n_experts"], m["top_k"])
        assert (c.h, c.hs) == (s["expert_hidden"], s["shared_hidden"])
        assert c.N * c.h * c.l == s["n_experts"] * s["expert_hidden"] * s["latent"]
