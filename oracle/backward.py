"""Float64 CPU oracle of the LatentMoE layer backward pass: the gradients of a
loss L with respect to the layer input and weights, given G = dL/dy.

TEST INFRASTRUCTURE ONLY (as oracle/lmoe.py): imported by the tests and by
nothing on the product path; it shares no code with the CUDA library.

What it differentiates is the forward of oracle/lmoe.py, the layer of
"NVIDIA Nemotron 3: Efficient and Open Intelligence" (xllm-io review),
section 三 eq.(1) and section 五, with the router of "Nemotron-3 Super 精读报告"
table 6.3 (Sigmoid + Expert Biasing).  The pages train this layer (the same
report, section 6: AdamW, an aux-loss-free balancing strategy with update
rate 1e-3) but print no backward formulas; the gradient of a fixed function
is its exact derivative, taken here step by step in reverse order of the
forward (chain rule), per token:

  forward                          backward
  z = W_r x, s = sigmoid(z)        dz_e = ds_e s_e (1 - s_e)   (selected e only)
  w_k = s_Sk / Z, Z = sum s_S      ds_Sk = (dw_k - sum_j w_j dw_j) / Z
  u = W_dn x                       dx += W_dn^T du,   dW_dn += du x^T
  a_k = W1[e] u, g_k = sqrelu(a_k) da_k = dg_k * 2 max(a_k, 0)
                                   du += W1[e]^T da_k, dW1[e] += da_k u^T
  o_k = W2[e] g_k                  dg_k = W2[e]^T do_k, dW2[e] += do_k g_k^T
  v = sum_k w_k o_k                do_k = w_k dv,       dw_k = dv . o_k
  r = W_upl v                      dv = W_upl^T G,      dW_upl += G v^T
  hs = sqrelu(W_s1 x)              dhs_pre = (W_s2^T G) * 2 max(W_s1 x, 0)
  sh = W_s2 hs                     dW_s2 += G hs^T,     dW_s1 += dhs_pre x^T
  y = r + sh                       dx += W_s1^T dhs_pre + W_r^T dz

Readings taken where the pages are silent:
  * the top-K selection is piecewise constant in z: its derivative is zero
    wherever the selected set does not change (everywhere except on ties),
    so gradients reach the router only through the weights w;
  * the expert bias b enters the selection only and so gets no gradient; it
    moves by the aux-loss-free update of bias_update instead;
  * sqrelu'(0) = 0 (the two one-sided derivatives agree there).
"""
from __future__ import annotations

from typing import Callable, Dict, Optional

import numpy as np

from .lmoe import route, sqrelu

__all__ = ["layer_backward", "expert_backward", "router_backward", "bias_update",
           "BIAS_UPDATE_RATE"]

# "Nemotron-3 Super 精读报告", table 6.3: update rate of the aux-loss-free
# balancing strategy
BIAS_UPDATE_RATE = 1e-3


def expert_backward(U: np.ndarray, dV: np.ndarray, w: np.ndarray, W1e: np.ndarray,
                    W2e: np.ndarray) -> Dict[str, np.ndarray]:
    """One expert's part of the backward, over the n routed rows that chose it.

    U [n][l]: the rows' expert inputs u; dV [n][l]: dL/dv of the rows' tokens;
    w [n]: the rows' router weights; W1e [h][l], W2e [l][h].  Per row (the
    expert lines of the table above): a = W1e u, g = sqrelu(a), o = W2e g,
    dw = dv . o, do = w dv, dW2e = sum do g^T, da = (W2e^T do) * 2 max(a, 0),
    dW1e = sum da u^T, du = W1e^T da.
    Returns o [n][l], dw [n], dW1 [h][l], dW2 [l][h], du [n][l], and the
    factors of the weight gradients: do [n][l], g [n][h], da [n][h].
    """
    a = U @ W1e.T                                        # [n][h]
    g = sqrelu(a)
    o = g @ W2e.T                                        # [n][l]
    dw = np.sum(dV * o, axis=1)
    do = w[:, None] * dV                                 # [n][l]
    dW2 = do.T @ g
    da = (do @ W2e) * 2.0 * np.maximum(a, 0.0)           # [n][h]
    return {"o": o, "dw": dw, "dW1": da.T @ U, "dW2": dW2, "du": da @ W1e, "do": do, "g": g,
            "da": da}


def router_backward(s_sel: np.ndarray, dw: np.ndarray, S: np.ndarray, N: int) -> np.ndarray:
    """dL/dz [T][N] through the renormalised weights (the router lines of the
    table above): s_sel [T][K] the selected experts' scores, dw [T][K] =
    dL/dw, S [T][K] the selected experts; zero at the unselected experts."""
    Z = s_sel.sum(axis=1)
    w = s_sel / Z[:, None]
    ds_sel = (dw - np.sum(w * dw, axis=1, keepdims=True)) / Z[:, None]
    dz = np.zeros((S.shape[0], N), dtype=np.float64)
    np.put_along_axis(dz, S, ds_sel * s_sel * (1.0 - s_sel), axis=1)
    return dz


def layer_backward(x: np.ndarray, W_r: np.ndarray, bias: Optional[np.ndarray],
                   W_dn: Optional[np.ndarray], get_w1: Callable[[int], np.ndarray],
                   get_w2: Callable[[int], np.ndarray], W_upl: Optional[np.ndarray],
                   W_s1: np.ndarray, W_s2: np.ndarray, K: int, G: np.ndarray,
                   S: Optional[np.ndarray] = None) -> Dict[str, object]:
    """Gradients of L with respect to x and every weight, given G = dL/dy.

    Arguments as oracle.lmoe.layer_forward (float64, [out][in] weights; W_dn =
    W_upl = None is the standard MoE with u = x and r = v), plus G [T][d].
    S [T][K] optionally fixes the selected experts (the oracle's own top-K
    otherwise); the weights w are always renormalised from the oracle's own
    sigmoid scores.
    Returns dx [T][d], dW_r [N][d], dW_dn [l][d], dW_upl [d][l], dW_s1
    [h_s][d], dW_s2 [d][h_s] (dW_dn, dW_upl None for the standard MoE), and
    dW1, dW2: dicts expert -> [h][l], [l][h] over the experts some token
    selected (the others have zero gradient), plus S, w, dw [T][K] (dL/dw),
    dz [T][N] (dL/dz), and du, dv [T][l] (dL/du, dL/dv).
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    G = np.atleast_2d(np.asarray(G, dtype=np.float64))
    T, d = x.shape
    N = W_r.shape[0]
    latent = W_dn is not None
    # forward quantities the derivative needs
    z = x @ W_r.T
    S_own, _, _, s = route(z, bias, K)
    S = S_own if S is None else np.asarray(S, dtype=np.int64)
    s_sel = np.take_along_axis(s, S, axis=1)            # [T][K]
    Z = s_sel.sum(axis=1)                                # [T]
    w = s_sel / Z[:, None]
    u = x @ W_dn.T if latent else x.copy()
    hs_pre = x @ W_s1.T
    hs = sqrelu(hs_pre)

    # shared expert and up-projection
    dv = G @ W_upl if latent else G.copy()              # [T][l]
    dW_s2 = G.T @ hs
    dhs_pre = (G @ W_s2) * 2.0 * np.maximum(hs_pre, 0.0)
    dW_s1 = dhs_pre.T @ x
    dx = dhs_pre @ W_s1

    # experts, one selected expert at a time over the tokens that chose it
    du = np.zeros_like(u)
    dw = np.zeros((T, K), dtype=np.float64)
    dW1: Dict[int, np.ndarray] = {}
    dW2: Dict[int, np.ndarray] = {}
    v = np.zeros_like(u)
    for e in np.unique(S):
        e = int(e)
        tok, slot = np.nonzero(S == e)
        ex = expert_backward(u[tok], dv[tok], w[tok, slot], get_w1(e), get_w2(e))
        v[tok] += w[tok, slot][:, None] * ex["o"]
        dw[tok, slot] = ex["dw"]
        dW2[e] = ex["dW2"]
        dW1[e] = ex["dW1"]
        # a token selects e at most once, so tok has no repeats here
        du[tok] += ex["du"]
    dW_upl = G.T @ v if latent else None
    if latent:
        dW_dn = du.T @ x
        dx += du @ W_dn
    else:
        dW_dn = None
        dx += du

    # router: through the renormalised weights of the selected experts
    dz = router_backward(s_sel, dw, S, N)
    dW_r = dz.T @ x
    dx += dz @ W_r
    return {"dx": dx, "dW_r": dW_r, "dW_dn": dW_dn, "dW1": dW1, "dW2": dW2,
            "dW_upl": dW_upl, "dW_s1": dW_s1, "dW_s2": dW_s2, "S": S, "w": w,
            "dw": dw, "dz": dz, "du": du, "dv": dv}


def bias_update(bias: np.ndarray, counts: np.ndarray,
                rate: float = BIAS_UPDATE_RATE) -> np.ndarray:
    """Aux-loss-free load balancing: b_e <- b_e + rate * sign(mean - c_e).

    "Nemotron-3 Super 精读报告", table 6.3 names the strategy and its update
    rate (1e-3) but not the rule; the reading is the plain one for a bias
    that only steers selection: every expert that took more than the mean
    number of routed rows c_e in the batch loses `rate`, every expert below
    it gains `rate`, an expert exactly at the mean keeps its bias.
    Arithmetic in float32, as the bias is stored: b + f32(rate) * sign.
    """
    b = np.asarray(bias, dtype=np.float32)
    c = np.asarray(counts, dtype=np.int64)
    N = c.shape[0]
    total = int(c.sum())
    # compare N * c_e with the total: mean - c_e without rounding
    sign = np.sign(total - N * c).astype(np.float32)
    return (b + np.float32(rate) * sign).astype(np.float32)
