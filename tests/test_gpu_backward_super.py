"""Backward parity at the Super dims ("Nemotron-3 Super 精读报告", table 2.2:
d=4096, l=1024, N=512, K=22, h=2688, h_s=5376), at the decode (T=256) and
prefill (T=8192, Zipf router bias) batches, in the launch configuration the
training-step benchmark times.

The weight gradients are sums over every token, and the float64 oracle cannot
run the whole expert pass of 8192 tokens in a test, so two passes share one
layer:

  * dL/dy dense (the benchmark's upstream gradient):
      - dx on 16 sampled tokens (first and last included): dx of a token
        depends on that token only, so the oracle runs on those tokens;
      - 16 sampled rows of dW_s1 and columns of dW_s2, exact over all T
        tokens from a few columns of the shared expert;
      - dW1[e], dW2[e] in full for the expert with the most rows, one with
        the fewest, and one without rows (exactly zero): one expert's
        backward over all of its rows (oracle.backward.expert_backward);
  * dL/dy zero except on the sampled tokens: every gradient of the layer is
    then a sum over those tokens alone, so all of them are compared in full
    (dx, dW_r, dW_dn, dW_upl, dW_s1, dW_s2, and dW1, dW2 of every expert the
    tokens chose); every other expert's gradient, and dx of every other
    token, must be exactly zero.

An expert's weight gradient here sums one or two routed rows: an outer
product a b^T whose elements carry the whole error of both factors, with no
averaging over rows.  Each factor is a bf16 intermediate under the error
model of tests/_parity.py, |da| <= 2^-7 (|a| + k RMS(a)) with k = 3e-2 / 2^-7
= 3.84, so |d(a b^T)| <= 2^-6 (|a| + k RMS(a)) (|b| + k RMS(b)), summed over
the rows: that is the elementwise bound of these gradients (for dW1 the
factors are da and u, for dW2 do and g), with the relative RMS bar of the
other gradients over all chosen experts.

The GPU's routing is checked first: equal to the oracle's for every token
whose K-th vs (K+1)-th key gap exceeds 1e-3, a valid top-K otherwise; the
oracle then differentiates with the GPU's selected experts.  Bars: those of
tests/test_gpu_backward.py (derived there from the bf16 roundings).
"""
import numpy as np
import pytest
import torch

from oracle import backward as B
from oracle import lmoe as O
from tests._parity import GAP, elem_ok, make, to64
from tests.test_gpu_backward import (ABS_RMS, EXPERT_ABS_RMS, REL_ELEM, RMS_BAR,
                                     ROUTER_ABS_RMS, ROUTER_RMS_BAR)

pytestmark = pytest.mark.gpu

N_SAMPLE = 16
K_TAIL = 3e-2 / 2.0 ** -7    # the tail term of a bf16 intermediate, in units of 2^-7 RMS


def _bars(name):
    if name == "dW_r":
        return ROUTER_RMS_BAR, ROUTER_ABS_RMS
    if name.startswith(("dW1", "dW2")):
        return RMS_BAR, EXPERT_ABS_RMS
    return RMS_BAR, ABS_RMS


def _compare(report, name, got, want):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{name}: unwritten or non-finite elements"
    rb, ab = _bars(name)
    ok, ratio, rr = elem_ok(got, want, rel=REL_ELEM, abs_rms=ab, rel_rms=rb)
    report[name] = (round(rr, 5), round(ratio, 3))
    assert ok, f"{name}: RMS rel {rr:.3g}, elementwise error {ratio:.3g} x bound"


@pytest.fixture(scope="module", params=["super_decode", "super_prefill"])
def layer_case(request):
    from lmoe_synth import CONFIGS
    cfg = CONFIGS[request.param]
    w, x, layer = make(cfg, backward=True)
    yield cfg, w, x, layer
    layer.close()
    del w, x, layer
    torch.cuda.empty_cache()


def _factor_ratio(got, want, factors):
    """Worst elementwise error over the bound of a sum of few outer products
    a_r b_r^T: 2^-6 sum_r (|a_r| + k RMS(a_r)) (|b_r| + k RMS(b_r))."""
    a, b = factors
    bound = np.zeros((a.shape[1], b.shape[1]))
    for r in range(a.shape[0]):
        ka = np.abs(a[r]) + K_TAIL * np.sqrt(np.mean(a[r] ** 2))
        kb = np.abs(b[r]) + K_TAIL * np.sqrt(np.mean(b[r] ** 2))
        bound += np.outer(ka, kb)
    bound *= 2.0 ** -6
    return float(np.max(np.abs(got - want) / np.maximum(bound, 1e-300)))


def _run_backward(layer, x, dy):
    layer.forward(x)
    grads = layer.grad_buffers()
    for g in grads.values():
        g.fill_(float("nan"))          # every element must be written
    dx = layer.backward(x, dy, grads)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    return grads, dx


def _routing(cfg, layer, x64, Wr, b):
    """The GPU's selected experts, checked against the oracle's routing; and
    the oracle's scores (the weights renormalise them over the GPU's set)."""
    S = layer.debug("topk_idx").numpy().astype(np.int64)
    S_o, _, gap, s = O.route(x64 @ Wr.T, b, cfg.K)
    key = s + b[None, :]
    clear = gap > GAP
    assert np.array_equal(np.sort(S[clear], 1), np.sort(S_o[clear], 1))
    for t in np.nonzero(~clear)[0]:
        assert O.is_valid_topk(key[t], S[t], GAP), f"token {t}: invalid top-K"
    return S, s


def _sample_tokens(T, seed):
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, T - 1), N_SAMPLE - 2, replace=False)
    return np.sort(np.concatenate([[0, T - 1], mid]))


def test_backward_super_dims(layer_case):
    from lmoe_synth import make_grad_out
    cfg, w, x, layer = layer_case
    T, K, N = cfg.T, cfg.K, cfg.N
    W = {k: to64(w[k]) for k in ("w_router", "router_bias", "w_dn", "w_upl", "w_s1", "w_s2")}
    get_w1 = lambda e: to64(w["w1"][e])  # noqa: E731
    get_w2 = lambda e: to64(w["w2"][e])  # noqa: E731
    x64 = to64(x)
    dy = make_grad_out(cfg, T=T, device="cuda")
    G = to64(dy)
    toks = _sample_tokens(T, 1000 + cfg.seed)

    # ---- dL/dy dense ------------------------------------------------------
    grads, dx = _run_backward(layer, x, dy)
    S, s = _routing(cfg, layer, x64, W["w_router"], W["router_bias"])
    ref = B.layer_backward(x64[toks], W["w_router"], W["router_bias"], W["w_dn"], get_w1,
                           get_w2, W["w_upl"], W["w_s1"], W["w_s2"], K, G[toks], S=S[toks])
    report = {}
    _compare(report, "dx[sampled tokens]", to64(dx)[toks], ref["dx"])
    rng = np.random.default_rng(2000 + cfg.seed)
    J = np.sort(rng.choice(cfg.hs, N_SAMPLE, replace=False))
    hs_pre = x64 @ W["w_s1"][J].T                                   # [T][16]
    dhs_pre = (G @ W["w_s2"][:, J]) * 2.0 * np.maximum(hs_pre, 0.0)
    _compare(report, "dW_s1[sampled rows]", to64(grads["d_s1"][torch.as_tensor(J).cuda()]),
             dhs_pre.T @ x64)
    _compare(report, "dW_s2[sampled cols]",
             to64(grads["d_s2"][:, torch.as_tensor(J).cuda()]),
             G.T @ O.sqrelu(hs_pre))
    counts = np.bincount(S.reshape(-1), minlength=N)
    e_big = int(np.argmax(counts))
    e_small = int(np.argmin(np.where(counts > 0, counts, np.iinfo(np.int64).max)))
    dv = G @ W["w_upl"]
    for tag, e in (("largest", e_big), ("smallest", e_small)):
        tok, slot = np.nonzero(S == e)
        s_sel = np.take_along_axis(s[tok], S[tok], axis=1)
        w_rows = s[tok, e] / s_sel.sum(axis=1)
        U = x64[tok] @ W["w_dn"].T
        ex = B.expert_backward(U, dv[tok], w_rows, get_w1(e), get_w2(e))
        if len(tok) > 4:
            _compare(report, f"dW1[{tag} segment, {len(tok)} rows]", to64(grads["d_w1"][e]),
                     ex["dW1"])
            _compare(report, f"dW2[{tag} segment, {len(tok)} rows]", to64(grads["d_w2"][e]),
                     ex["dW2"])
        else:
            # a few rows: the outer-product bound of the dL/dy-on-samples pass
            r1 = _factor_ratio(to64(grads["d_w1"][e]), ex["dW1"], (ex["da"], U))
            r2 = _factor_ratio(to64(grads["d_w2"][e]), ex["dW2"], (ex["do"], ex["g"]))
            report[f"dW1, dW2 [{tag} segment, {len(tok)} rows] factor bound"] = (round(r1, 3),
                                                                                 round(r2, 3))
            assert r1 <= 1.0 and r2 <= 1.0, (r1, r2)
    empty = np.nonzero(counts == 0)[0]
    if cfg.bias == "zipf":
        assert len(empty) > 0, "the Zipf bias leaves some experts without rows"
    for e in empty[:3]:
        assert not grads["d_w1"][int(e)].any() and not grads["d_w2"][int(e)].any()
    print(cfg.name, "dense dy", report, "counts max/min>0:", counts.max(),
          counts[counts > 0].min(), "empty experts:", len(empty))
    del grads, dx

    # ---- dL/dy only on the sampled tokens ----------------------------------
    mask = torch.zeros((T, 1), dtype=torch.bfloat16, device="cuda")
    mask[torch.as_tensor(toks).cuda()] = 1
    dy_s = dy * mask
    grads, dx = _run_backward(layer, x, dy_s)
    assert np.array_equal(layer.debug("topk_idx").numpy().astype(np.int64), S)
    report = {}
    dx64 = to64(dx)
    others = np.setdiff1d(np.arange(T), toks)
    assert not np.any(dx64[others]), "dx of a token with zero dL/dy must be zero"
    _compare(report, "dx", dx64[toks], ref["dx"])
    # the router gradient has a row per expert: rows of experts no sampled
    # token chose are exactly zero, the rest compared (zero rows would only
    # dilute the RMS of the bound's tail term)
    reached = np.unique(S[toks])
    gr = to64(grads["d_router"])
    assert not np.any(np.delete(gr, reached, axis=0)), "router rows of unchosen experts"
    _compare(report, "dW_r", gr[reached], ref["dW_r"][reached])
    for name, key in (("dW_dn", "d_dn"), ("dW_upl", "d_upl"), ("dW_s1", "d_s1"),
                      ("dW_s2", "d_s2")):
        _compare(report, name, to64(grads[key]), ref[name])
    chosen = sorted(ref["dW1"].keys())
    for name, key in (("dW1", "d_w1"), ("dW2", "d_w2")):
        sq_err, sq_ref = 0.0, 0.0
        for e in chosen:
            got = to64(grads[key][e])
            assert np.isfinite(got).all(), f"{name}[{e}]: non-finite"
            sq_err += float(np.sum((got - ref[name][e]) ** 2))
            sq_ref += float(np.sum(ref[name][e] ** 2))
        rr = (sq_err / sq_ref) ** 0.5
        report[name + "[chosen] rms rel"] = round(rr, 5)
        assert rr <= RMS_BAR, f"{name}[chosen]: RMS rel {rr:.3g}"
    # elementwise, from the factors of the few rows of each expert: the
    # experts with the most sampled rows and a random few
    dv = G @ W["w_upl"]
    rows_of = {e: np.nonzero((S[toks] == e).any(axis=1))[0] for e in chosen}
    by_rows = sorted(chosen, key=lambda e: -len(rows_of[e]))
    pick = by_rows[:4] + list(np.random.default_rng(3000 + cfg.seed).choice(by_rows[4:], 8,
                                                                          replace=False))
    worst = {"dW1": 0.0, "dW2": 0.0}
    for e in pick:
        tk = toks[rows_of[e]]
        s_sel = np.take_along_axis(s[tk], S[tk], axis=1)
        U = x64[tk] @ W["w_dn"].T
        ex = B.expert_backward(U, dv[tk], s[tk, e] / s_sel.sum(axis=1), get_w1(e), get_w2(e))
        worst["dW1"] = max(worst["dW1"], _factor_ratio(to64(grads["d_w1"][e]), ex["dW1"],
                                                       (ex["da"], U)))
        worst["dW2"] = max(worst["dW2"], _factor_ratio(to64(grads["d_w2"][e]), ex["dW2"],
                                                       (ex["do"], ex["g"])))
    report["dW1, dW2 factor bound (worst ratio)"] = {k: round(v, 3) for k, v in worst.items()}
    assert worst["dW1"] <= 1.0 and worst["dW2"] <= 1.0, worst
    nz1 = grads["d_w1"].reshape(N, -1).abs().amax(1).cpu().numpy()
    nz2 = grads["d_w2"].reshape(N, -1).abs().amax(1).cpu().numpy()
    rest = np.setdiff1d(np.arange(N), chosen)
    assert not nz1[rest].any() and not nz2[rest].any(), \
        "an expert no sampled token chose has a nonzero gradient"
    print(cfg.name, "sampled dy", report, "experts chosen:", len(chosen))
