"""Float64 CPU oracle of the LatentMoE layer forward pass.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously correct
statement of what the layer computes.  It is imported by the tests, by the
smoke check and by the CPU-baseline leg of the benchmark, and by nothing on
the product path; it shares no code with the CUDA library.

Sources (web pages on NVIDIA Nemotron 3):
  [R1] "NVIDIA Nemotron 3: Efficient and Open Intelligence" (xllm-io paper
       review), section 三 "LatentMoE 架构", eq.(1) and the paragraph after it;
       section 五 "架构实现要点".
  [R5] "Nemotron-3 Super 精读报告" (tuntang.top deep reading), table 2.2
       (架构配置详表), section 3.3 (Latent 投影解法), table 6.3 (超参数:
       路由机制 "Sigmoid + Expert Biasing").
  [R2] "Nemotron 3全新混合專家架構，推理效率升4倍" (digipub), section
       "LatentMoE".

The layer, per token x_t (hidden width d):
  1. router logits z = W_r x_t at width d, scores s = sigmoid(z) and keys
     key = s + b (the expert-biasing term of the router) [R5 table 6.3;
     R1 sec. 五: gating stays at d];
  2. the K experts with the largest key (descending, ties to the lower
     expert id) and weights w_k = s_k / sum_k' s_k' (renormalised to sum 1);
  3. u = W_dn x_t, projection d -> l [R1 sec. 三; R2 "LatentMoE"];
  4. each selected expert runs in latent space: o_k = W2[e] sqrelu(W1[e] u)
     with sqrelu(a) = max(a, 0)^2 (the activation is a stated convention:
     the pages do not name one);
  5. v = sum_k w_k o_k in latent space, then one projection back r = W_upl v
     (exact by linearity of W_upl) [R1 sec. 三];
  6. shared expert at width d: sh = W_s2 sqrelu(W_s1 x_t) [R1 sec. 三, "保留
     在原始维度 d 的非路由计算"; R5 table 2.2 "Shared Expert Intermediate Size"];
  7. y = r + sh.

Readings taken where the pages are silent:
  * the bias b enters the selection only; weights use the unbiased s;
  * ties in key go to the lower expert id, and slot order is key-descending;
  * no biases in the linear layers [R5 sec. 2.3 "无 Dropout 和 Bias"].
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Optional

import numpy as np

__all__ = [
    "sigmoid", "sqrelu", "route", "segments", "expert_ffn", "layer_forward",
    "token_forward", "scaling_relation", "is_valid_topk",
]


def sigmoid(z: np.ndarray) -> np.ndarray:
    """Logistic function in float64 (router score, R5 table 6.3)."""
    z = np.asarray(z, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-z))


def sqrelu(a: np.ndarray) -> np.ndarray:
    """Squared ReLU, max(a, 0)^2 (the expert and shared-expert activation)."""
    a = np.asarray(a, dtype=np.float64)
    return np.square(np.maximum(a, 0.0))


def route(z: np.ndarray, bias: Optional[np.ndarray], K: int):
    """Sigmoid router with expert biasing and top-K renormalisation.

    z: [T][N] float64 logits; bias: [N] or None (zeros); K: experts per token.
    Returns (S, w, gap, s):
      S   [T][K] int64, the selected experts, key-descending, ties to lower id;
      w   [T][K] float64, s_S / sum(s_S)  (sums to 1 per token);
      gap [T]    float64, key of the K-th minus key of the (K+1)-th expert
                 (+inf when K == N);
      s   [T][N] float64 sigmoid scores.
    Follows R5 table 6.3 (Sigmoid + Expert Biasing) and R1 eq.(1) (K' active
    experts per token).
    """
    z = np.atleast_2d(np.asarray(z, dtype=np.float64))
    T, N = z.shape
    if not (1 <= K <= N):
        raise ValueError("need 1 <= K <= N")
    b = np.zeros(N) if bias is None else np.asarray(bias, dtype=np.float64)
    s = sigmoid(z)
    key = s + b[None, :]
    ids = np.arange(N)
    S = np.empty((T, K), dtype=np.int64)
    gap = np.empty(T, dtype=np.float64)
    for t in range(T):
        # primary: key descending; secondary: expert id ascending
        order = np.lexsort((ids, -key[t]))
        S[t] = order[:K]
        gap[t] = key[t, order[K - 1]] - key[t, order[K]] if K < N else math.inf
    sel = np.take_along_axis(s, S, axis=1)
    w = sel / sel.sum(axis=1, keepdims=True)
    return S, w, gap, s


def is_valid_topk(key_row: np.ndarray, chosen: np.ndarray, eps: float) -> bool:
    """True when `chosen` (K distinct ids) is a top-K set of `key_row` up to eps.

    A set is valid when every chosen key is >= every unchosen key - eps.  Used
    only where several answers are correct (keys closer than the comparison
    precision); the oracle's own set is always valid with eps = 0.
    """
    key_row = np.asarray(key_row, dtype=np.float64)
    chosen = np.asarray(chosen, dtype=np.int64)
    if len(set(chosen.tolist())) != len(chosen):
        return False
    mask = np.zeros(key_row.shape[0], dtype=bool)
    mask[chosen] = True
    if mask.all():
        return True
    return bool(key_row[mask].min() >= key_row[~mask].max() - eps)


def segments(S: np.ndarray, N: int):
    """Per-expert segments of the routed rows (a stable counting sort).

    Row order: expert ascending, then token ascending (then slot, which never
    ties because a token selects an expert at most once).
    Returns counts [N], offsets [N+1] (exclusive scan), perm [T*K] (row ->
    t*K + k) and inv [T][K] (slot -> row).
    """
    S = np.asarray(S, dtype=np.int64)
    T, K = S.shape
    counts = np.bincount(S.reshape(-1), minlength=N).astype(np.int64)
    offsets = np.zeros(N + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.empty(T * K, dtype=np.int64)
    inv = np.empty((T, K), dtype=np.int64)
    fill = offsets[:-1].copy()
    for t in range(T):
        for k in range(K):
            e = S[t, k]
            r = fill[e]
            fill[e] += 1
            perm[r] = t * K + k
            inv[t, k] = r
    return counts, offsets, perm, inv


def expert_ffn(U: np.ndarray, W1e: np.ndarray, W2e: np.ndarray) -> np.ndarray:
    """Latent-space expert: rows of U [n][l] -> W2e sqrelu(W1e u)  ([n][l])."""
    return sqrelu(U @ W1e.T) @ W2e.T


def _expert_quantisers(quant: Dict):
    """(q_u, q_w, q_h): quantise-dequantise maps of the expert inputs u, an
    expert weight matrix and the expert hidden activation, for the NVFP4
    ("fmt" absent or "nvfp4") or the FP8 W8A8 ("fmt": "fp8") expert layer."""
    if quant.get("fmt", "nvfp4") == "w4a16":
        # NVFP4 weights, unquantised (16-bit) activations
        from . import nvfp4
        wq = dict(block2d=quant.get("w2d", False), mse=quant.get("wmse", False))
        return (lambda a: a,
                lambda W: nvfp4.fake_quant(W, nvfp4.weight_global_scale(W), **wq),
                lambda a: a)
    if quant.get("fmt", "nvfp4") == "fp8":
        from . import fp8
        return (lambda a: fp8.fake_quant(a, quant["s_u"]),
                lambda W: fp8.fake_quant(W, fp8.weight_scale(W)),
                lambda a: fp8.fake_quant(a, quant["s_h"]))
    from . import nvfp4
    wq = dict(block2d=quant.get("w2d", False), mse=quant.get("wmse", False))
    return (lambda a: nvfp4.fake_quant(a, quant["g_u"]),
            lambda W: nvfp4.fake_quant(W, nvfp4.weight_global_scale(W), **wq),
            lambda a: nvfp4.fake_quant(a, quant["g_h"]))


def layer_forward(x: np.ndarray, W_r: np.ndarray, bias: Optional[np.ndarray],
                  W_dn: Optional[np.ndarray], get_w1: Callable[[int], np.ndarray],
                  get_w2: Callable[[int], np.ndarray], W_upl: Optional[np.ndarray],
                  W_s1: np.ndarray, W_s2: np.ndarray, K: int,
                  quant: Optional[Dict] = None) -> Dict[str, np.ndarray]:
    """The LatentMoE layer forward pass for the tokens in x ([T][d], float64).

    Weights are [out][in] float64: W_r [N][d], W_dn [l][d], W_upl [d][l],
    W_s1 [h_s][d], W_s2 [d][h_s]; get_w1(e) -> [h][l], get_w2(e) -> [l][h].
    W_dn = W_upl = None is the standard MoE layer that the pages compare
    LatentMoE against ("NVIDIA Nemotron 3: Efficient and Open Intelligence",
    section 三 eq.(1) and section 六 Table 1): no projections, the experts
    work at width l = d on x itself, u = x and r = v.
    Every token is computed independently, so any subset of tokens may be
    passed.  quant: None for the BF16 layer, or a dict with the NVFP4 global
    scales {"g_u": float, "g_h": float} for the NVFP4-expert layer, in which
    u, W1[e], W2[e] and the expert hidden activation are replaced by their
    NVFP4 quantise-dequantise images (oracle.nvfp4); optional "w2d" and
    "wmse" (bool) select 2D 16x16 weight blocks and MSE-searched weight
    block scales.  quant = {"fmt": "fp8", "s_u": float, "s_h": float} is the
    FP8 W8A8 expert layer (oracle.fp8: E4M3, per-tensor scales);
    {"fmt": "w4a16"} (with optional "w2d", "wmse") has NVFP4 weights and
    unquantised activations.

    Returns a dict with S, w, gap, s, z, u, v, r, hs, sh, y (float64); hs is
    the shared expert's hidden activation sqrelu(W_s1 x).
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    if (W_dn is None) != (W_upl is None):
        raise ValueError("W_dn and W_upl are both given (LatentMoE) or both None")
    T = x.shape[0]
    N = W_r.shape[0]
    l = x.shape[1] if W_dn is None else W_dn.shape[0]
    # 1-2: router at width d
    z = x @ W_r.T
    S, w, gap, s = route(z, bias, K)
    # 3: latent down-projection (none for the standard MoE)
    u = x.copy() if W_dn is None else x @ W_dn.T
    if quant is not None:
        q_u, q_w, q_h = _expert_quantisers(quant)
        u_in = q_u(u)
    else:
        u_in = u
    # 4-5: experts in latent space, weighted sum in latent space
    v = np.zeros((T, l), dtype=np.float64)
    for e in np.unique(S):
        tok, slot = np.nonzero(S == e)
        W1e = get_w1(int(e))
        W2e = get_w2(int(e))
        if quant is not None:
            W1e, W2e = q_w(W1e), q_w(W2e)
            g = q_h(sqrelu(u_in[tok] @ W1e.T))
            o = g @ W2e.T
        else:
            o = expert_ffn(u_in[tok], W1e, W2e)
        # a token selects e at most once, so tok has no repeats here
        v[tok] += w[tok, slot][:, None] * o
    # 5: one projection back to width d (none for the standard MoE)
    r = v.copy() if W_upl is None else v @ W_upl.T
    # 6: shared expert at width d
    hs = sqrelu(x @ W_s1.T)
    sh = hs @ W_s2.T
    return {"S": S, "w": w, "gap": gap, "s": s, "z": z, "u": u, "v": v,
            "r": r, "hs": hs, "sh": sh, "y": r + sh}


def token_forward(x_t: np.ndarray, S_t: np.ndarray, s_t: np.ndarray,
                  W_dn: np.ndarray, get_w1, get_w2, W_upl: np.ndarray,
                  quant: Optional[Dict] = None) -> Dict[str, np.ndarray]:
    """Routed branch of one token for a given expert set S_t.

    Used where the top-K set is not unique at the comparison precision (near
    ties): the caller first checks with is_valid_topk that S_t is a top-K set
    under the oracle's own keys.  Weights are renormalised from the oracle's
    scores s_t.  Returns v [l] and r [d].  W_dn = W_upl = None: the standard
    MoE (u = x, r = v), as in layer_forward.
    """
    x_t = np.asarray(x_t, dtype=np.float64).reshape(-1)
    S_t = np.asarray(S_t, dtype=np.int64).reshape(-1)
    sel = np.asarray(s_t, dtype=np.float64)[S_t]
    w = sel / sel.sum()
    u = x_t.copy() if W_dn is None else W_dn @ x_t
    if quant is not None:
        q_u, q_w, q_h = _expert_quantisers(quant)
        u = q_u(u[None, :])[0]
    v = np.zeros(u.shape[0], dtype=np.float64)
    for k, e in enumerate(S_t):
        W1e = get_w1(int(e))
        W2e = get_w2(int(e))
        if quant is not None:
            W1e, W2e = q_w(W1e), q_w(W2e)
            g = q_h(sqrelu(W1e @ u)[None, :])[0]
            o = W2e @ g
        else:
            o = W2e @ sqrelu(W1e @ u)
        v += w[k] * o
    return {"v": v, "r": v.copy() if W_upl is None else W_upl @ v, "w": w}


def scaling_relation(N: int, K: int, d: int, l: int):
    """Eq.(1) of R1: N' = N d / l and K' = K d / l (exact when l divides N d)."""
    if (N * d) % l or (K * d) % l:
        raise ValueError("d/l does not scale N, K to integers")
    return N * d // l, K * d // l
