"""Helpers of the GPU parity tests: build a layer from a seeded workload, run
the oracle on a subset of its tokens, and compare.

Tolerances:
  * routing indices equal for every token whose oracle gap between the K-th
    and (K+1)-th key exceeds 1e-3 (the stated bar);
  * the layer output y within max|err| <= 2e-2 * RMS(y) over the compared
    tokens (the stated bar for BF16 experts);
  * intermediates (u, hs, v) and single-branch outputs, two derived bars:
      - RMS(err) <= 1e-2 RMS(ref): each value is stored in bf16 (relative
        rounding <= 2^-9) and carries the independent roundings of a few bf16
        upstream operands (x, u, H, O, v), so its relative RMS error is a few
        times 2^-9 (~0.4% measured for v); 1e-2 is ~5 x 2^-9;
      - elementwise |err| <= 2^-7 |ref| + 3e-2 RMS(ref): 2^-7 covers the
        element's own and its operands' roundings, 3e-2 RMS the tail of the
        accumulated upstream noise (max over ~1e4..1e5 elements of a noise
        with sigma ~ 2 x 2^-9 RMS is ~ 4.5 sigma ~ 1.8e-2 RMS).
    A plain max|err|/RMS bar does not fit heavy-tailed tensors: hs = sqrelu(.)
    has max/RMS ~ 13, so its bf16 storage alone costs ~ 0.025 RMS.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import lmoe as O

GAP = 1e-3
TOL_BF16 = 2e-2
REL_ELEM = 2.0 ** -7
ABS_RMS = 3e-2
REL_RMS = 1e-2
W_TOL = 1e-5


def to64(t):
    """float64 numpy copy of a tensor (None for a missing weight)."""
    if t is None:
        return None
    return t.detach().to("cpu").to(torch.float64).numpy()


def make(cfg, T=None, device="cuda", max_tokens=None, overrides=None, backward=False):
    """Seeded weights and x on the device, and the layer built from them."""
    from lmoe_synth import make_weights, make_x
    from latent_space_mixture_b200 import LatentMoE
    w, gen = make_weights(cfg, device=device)
    x = make_x(cfg, gen, T=T, device=device)
    if overrides:
        for k, fn in overrides.items():
            w[k] = fn(w[k])
    from lmoe_synth import act_global_scales
    layer = LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs,
                      max_tokens or x.shape[0], w, expert_format=cfg.fmt,
                      act_gscales=act_global_scales(cfg) if cfg.fmt != "bf16" else (0.0, 0.0),
                      projections=cfg.proj, nvfp4_weights=cfg.wq, backward=backward)
    return w, x, layer


def quant_of(cfg):
    """The oracle's quantisation settings for a workload (None for BF16)."""
    from lmoe_synth import act_global_scales
    if cfg.fmt == "bf16":
        return None
    g_u, g_h = act_global_scales(cfg)
    if cfg.fmt == "fp8":
        return {"fmt": "fp8", "s_u": float(np.float32(g_u)), "s_h": float(np.float32(g_h))}
    if cfg.fmt == "w4a16":
        return {"fmt": "w4a16", "w2d": cfg.wq in ("2d", "2d_mse"),
                "wmse": cfg.wq in ("mse", "2d_mse")}
    return {"g_u": float(np.float32(g_u)), "g_h": float(np.float32(g_h)),
            "w2d": cfg.wq in ("2d", "2d_mse"), "wmse": cfg.wq in ("mse", "2d_mse")}


def oracle_tokens(w, x_rows: torch.Tensor, K: int, quant=None):
    """The oracle on the given token rows, expert weights fetched (and up-cast)
    per expert on demand; nothing is cached, so host memory stays bounded."""

    def fetch(name, e):
        return to64(w[name][e])

    out = O.layer_forward(to64(x_rows), to64(w["w_router"]), to64(w["router_bias"]),
                          to64(w.get("w_dn")), lambda e: fetch("w1", e),
                          lambda e: fetch("w2", e), to64(w.get("w_upl")), to64(w["w_s1"]),
                          to64(w["w_s2"]), K, quant=quant)
    out["_fetch"] = fetch
    return out


def max_rel(a: np.ndarray, b: np.ndarray) -> float:
    """max|a - b| / RMS(b)."""
    rms = float(np.sqrt(np.mean(b * b)))
    return float(np.max(np.abs(a - b))) / (rms if rms > 0 else 1.0)


def rms_rel(a: np.ndarray, ref: np.ndarray) -> float:
    """RMS(a - ref) / RMS(ref)."""
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.sqrt(np.mean((a - ref) ** 2))) / (rms if rms > 0 else 1.0)


def elem_ok(a: np.ndarray, ref: np.ndarray, rel=REL_ELEM, abs_rms=ABS_RMS, rel_rms=REL_RMS):
    """The bf16 error model of an intermediate: relative RMS error and the
    elementwise tail bound.  Returns (ok, worst elementwise err / bound,
    relative RMS error)."""
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = rel * np.abs(ref) + abs_rms * rms
    ratio = float(np.max(np.abs(a - ref) / np.maximum(bound, 1e-300)))
    rr = rms_rel(a, ref)
    return ratio <= 1.0 and rr <= rel_rms, ratio, rr


def compare_layer(layer, w, x, y, tokens, K, tol=TOL_BF16, quant=None, elem_rel=REL_ELEM,
                  check_v=True):
    """Compare the last forward of `layer` (x -> y) with the oracle on `tokens`.

    Returns a dict of measured errors; asserts the bar.  Near-tie tokens whose
    GPU set differs from the oracle's must hold a valid top-K set under the
    oracle's keys (within GAP), and their outputs are compared with the
    oracle's for that set.
    """
    tokens = np.asarray(tokens)
    o = oracle_tokens(w, x[tokens], K, quant=quant)
    gi = layer.debug("topk_idx").numpy()[tokens]
    gw = layer.debug("topk_w").numpy()[tokens]
    key = o["s"] + to64(w["router_bias"])[None, :]
    v_ref = o["v"].copy()
    y_ref = o["y"].copy()
    n_tie_diff = 0
    for i in range(len(tokens)):
        same = sorted(gi[i].tolist()) == sorted(o["S"][i].tolist())
        if o["gap"][i] > GAP:
            assert same, f"token {tokens[i]}: routing {sorted(gi[i])} != {sorted(o['S'][i])}"
        if same:
            ref_w = dict(zip(o["S"][i].tolist(), o["w"][i].tolist()))
            for e, wv in zip(gi[i].tolist(), gw[i].tolist()):
                assert abs(wv - ref_w[e]) <= W_TOL, (tokens[i], e, wv, ref_w[e])
        else:
            n_tie_diff += 1
            assert O.is_valid_topk(key[i], gi[i], GAP), f"token {tokens[i]}: invalid top-K"
            tf = O.token_forward(to64(x[tokens[i]]), gi[i], o["s"][i], to64(w.get("w_dn")),
                                 lambda e: o["_fetch"]("w1", e), lambda e: o["_fetch"]("w2", e),
                                 to64(w.get("w_upl")), quant=quant)
            v_ref[i] = tf["v"]
            y_ref[i] = tf["r"] + o["sh"][i]
    # u is x itself without projections (the library keeps no copy of it)
    names = ("u", "hs", "v") if "w_dn" in w else ("hs", "v")
    got = {k: to64(layer.debug(k))[tokens] for k in names}
    ref = {"u": o["u"], "hs": o["hs"], "v": v_ref}
    errs = {"y_maxerr_over_rms": max_rel(to64(y)[tokens], y_ref),
            "near_tie_sets_differing": n_tie_diff}
    for k in names:
        ok, ratio, rr = elem_ok(got[k], ref[k], rel=elem_rel)
        errs[k + "_maxerr_over_rms"] = max_rel(got[k], ref[k])
        errs[k + "_err_over_bound"] = ratio
        errs[k + "_rms_rel"] = rr
        if k != "v" or check_v:
            assert ok, f"{k}: elementwise error {ratio:.3g} x bound, RMS rel error {rr:.3g}"
    assert errs["y_maxerr_over_rms"] <= tol, \
        f"y: max|err|/RMS = {errs['y_maxerr_over_rms']:.3g} > {tol}"
    return errs


def check_segments_valid(layer, T, N, K):
    """Properties of the per-expert segments that hold at any size."""
    idx = layer.debug("topk_idx").numpy().astype(np.int64)
    counts = layer.debug("counts").numpy().astype(np.int64)
    offsets = layer.debug("offsets").numpy().astype(np.int64)
    perm = layer.debug("perm").numpy().astype(np.int64)
    inv = layer.debug("inv").numpy().astype(np.int64)
    assert idx.min() >= 0 and idx.max() < N
    assert np.all(np.sort(idx, axis=1)[:, 1:] != np.sort(idx, axis=1)[:, :-1]), "duplicate expert"
    assert np.array_equal(counts, np.bincount(idx.reshape(-1), minlength=N))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    flat = idx.reshape(-1)
    assert np.array_equal(np.sort(perm), np.arange(T * K))
    assert np.array_equal(perm[inv.reshape(-1)], np.arange(T * K))
    # rows of each expert: that expert, ascending tokens
    seg_e = np.repeat(np.arange(N), counts)
    assert np.array_equal(flat[perm], seg_e)
    tok = perm // K
    same = seg_e[1:] == seg_e[:-1]
    assert np.all(tok[1:][same] > tok[:-1][same])
    return counts


# ---------------------------------------------------------------------------
# quantised layers at full size: the oracle's expert quantisers cost seconds
# per Super-width matrix, so each touched expert is quantised once, in a pool
# of spawned processes (never forked: the parent holds a CUDA context)

def _bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 values given as their 16-bit patterns -> float64 (exact)."""
    return (bits.astype(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _quantised_expert_rows(args):
    """Worker: one expert's quantised FFN on the latent rows U that chose it,
    as the oracle's own one-expert layer (N = 1, K = 1: every row takes the
    expert with weight 1; no projections, so its u is U itself; a zero-width
    shared expert contributes nothing).  Returns (e, o [n][l])."""
    e, w1_bits, w2_bits, U, quant = args
    W1e = _bf16_bits_to_f64(w1_bits)
    W2e = _bf16_bits_to_f64(w2_bits)
    l = U.shape[1]
    out = O.layer_forward(U, np.zeros((1, l)), None, None, lambda _: W1e, lambda _: W2e, None,
                          np.zeros((1, l)), np.zeros((l, 1)), 1, quant=quant)
    return e, out["v"]


def oracle_tokens_pooled(w, x_rows: torch.Tensor, K: int, quant, S_use: np.ndarray,
                         workers: int = 16):
    """The oracle layer on the given token rows with the selected experts
    S_use ([n][K], already checked to be a valid top-K set per token): the
    router, projections and shared expert as in oracle.lmoe.layer_forward,
    each expert's quantised FFN from _quantised_expert_rows, and
    v = sum_k w_k o_k with w renormalised from the oracle's scores."""
    import multiprocessing as mp
    x64 = to64(x_rows)
    z = x64 @ to64(w["w_router"]).T
    _, _, gap, s = O.route(z, to64(w["router_bias"]), K)
    S_use = np.asarray(S_use, dtype=np.int64)
    s_sel = np.take_along_axis(s, S_use, axis=1)
    wk = s_sel / s_sel.sum(axis=1, keepdims=True)
    u = x64 @ to64(w["w_dn"]).T
    jobs = []
    for e in np.unique(S_use):
        tok = np.nonzero((S_use == e).any(axis=1))[0]
        jobs.append((int(e), w["w1"][int(e)].view(torch.int16).cpu().numpy(),
                     w["w2"][int(e)].view(torch.int16).cpu().numpy(), u[tok], quant))
    v = np.zeros_like(u)
    with mp.get_context("spawn").Pool(min(workers, len(jobs))) as pool:
        for e, o in pool.imap_unordered(_quantised_expert_rows, jobs):
            tok, slot = np.nonzero(S_use == e)
            v[tok] += wk[tok, slot][:, None] * o
    hs = O.sqrelu(x64 @ to64(w["w_s1"]).T)
    y = v @ to64(w["w_upl"]).T + hs @ to64(w["w_s2"]).T
    return {"v": v, "y": y, "u": u, "hs": hs, "s": s, "gap": gap, "w": wk}


def compare_layer_pooled(layer, w, x, y, tokens, K, tol, quant):
    """compare_layer for quantised experts at full size, with the pooled
    oracle: routing checked first (equal outside the gap window, a valid
    top-K inside it), then y, u and hs against the oracle with the GPU's
    selected experts.  Returns the measured errors."""
    tokens = np.asarray(tokens)
    gi = layer.debug("topk_idx").numpy().astype(np.int64)[tokens]
    gw = layer.debug("topk_w").numpy()[tokens]
    z = to64(x[tokens]) @ to64(w["w_router"]).T
    S_o, w_o, gap, s = O.route(z, to64(w["router_bias"]), K)
    key = s + to64(w["router_bias"])[None, :]
    n_tie_diff = 0
    for i in range(len(tokens)):
        same = sorted(gi[i].tolist()) == sorted(S_o[i].tolist())
        if gap[i] > GAP:
            assert same, f"token {tokens[i]}: routing {sorted(gi[i])} != {sorted(S_o[i])}"
        if same:
            ref_w = dict(zip(S_o[i].tolist(), w_o[i].tolist()))
            for e, wv in zip(gi[i].tolist(), gw[i].tolist()):
                assert abs(wv - ref_w[e]) <= W_TOL, (tokens[i], e, wv, ref_w[e])
        else:
            n_tie_diff += 1
            assert O.is_valid_topk(key[i], gi[i], GAP), f"token {tokens[i]}: invalid top-K"
    o = oracle_tokens_pooled(w, x[tokens], K, quant, gi)
    errs = {"y_maxerr_over_rms": max_rel(to64(y)[tokens], o["y"]),
            "near_tie_sets_differing": n_tie_diff, "tokens": len(tokens)}
    for k in ("u", "hs"):
        got = to64(layer.debug(k))[tokens]
        ok, ratio, rr = elem_ok(got, o[k])
        errs[k + "_err_over_bound"] = ratio
        errs[k + "_rms_rel"] = rr
        assert ok, f"{k}: elementwise error {ratio:.3g} x bound, RMS rel error {rr:.3g}"
    got_v = to64(layer.debug("v"))[tokens]
    errs["v_rms_rel"] = rms_rel(got_v, o["v"])
    assert errs["y_maxerr_over_rms"] <= tol, \
        f"y: max|err|/RMS = {errs['y_maxerr_over_rms']:.3g} > {tol}"
    return errs
