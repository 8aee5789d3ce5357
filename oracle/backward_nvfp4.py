"""Float64 CPU oracle of the routed experts' backward pass under the NVFP4
training recipe.

TEST INFRASTRUCTURE ONLY (as oracle/lmoe.py): imported by the tests and by
nothing on the product path; it shares no code with the CUDA library.

Source: "Nemotron-3 Super 精读报告", section 5.3 (NVFP4 格式细节): weights are
quantised with 2D block scaling, gradients and activations with 1D blocks
along the GEMM reduction axis, a random Hadamard transform (RHT) is applied
to the inputs of the weight-gradient GEMMs and stochastic rounding to the
gradient tensors; table 5.2: the latent projections (and, in this build, the
router and the shared expert) stay BF16, so only the routed experts' GEMMs
take part.  The pages state the recipe, not its arithmetic.

Readings:
  * the forward is oracle.lmoe's NVFP4 expert layer with 2D weight blocks
    (one 16 x 16 block's scale serves W and its transpose, so the dgrad
    GEMMs reuse the forward's quantised weights W1q, W2q);
  * quantisers are identity in the derivative (straight-through): the
    backward differentiates the forward's arithmetic with the quantised
    values held fixed;
  * every GEMM of the backward takes NVFP4 operands, 1D blocks along its
    reduction axis:
      dgrad  dg = W2q^T Q_sr(do)    do = w dv, blocks along l
             du = W1q^T Q_sr(da)    da = dg * 2 max(a, 0), blocks along h
      wgrad  dW2[e] = Q_sr(R(do_e^T)) Q(R(g_e^T))^T   (reduction over the
             dW1[e] = Q_sr(R(da_e^T)) Q(R(u_e^T))^T    expert's routed rows)
    with Q_sr the stochastically rounding quantiser (gradients) and Q the
    round-to-nearest one (activations: g = sqrelu(a) quantised as in the
    forward, u the latent rows before quantisation), R the RHT on 16-row
    blocks of the token axis; an expert's rows are zero-padded to a multiple
    of 16 (zeros stay zeros under R and Q), and both operands of one wgrad
    GEMM take the same signs, so R^T R = I cancels in the product;
  * global scales: one per quantised tensor per call, amax / (6 * 448) over
    the whole tensor (all routed rows; after R for the wgrad operands);
  * random bits (oracle.nvfp4_train generators), one seed per tensor:
    seed + 0 do, + 1 da, + 2 the W2 wgrad's RHT, + 3 R(do^T), + 4 the W1
    wgrad's RHT, + 5 R(da^T); the wgrad operands are laid out [features]
    [padded rows of all experts, expert after expert], the element counter
    being row * width + column of that layout;
  * dL/dw_r = dv . o_r, with o_r the forward's expert output (the plain
    derivative; the router then follows oracle.backward).
"""
from __future__ import annotations

from typing import Callable, Dict

import numpy as np

from . import nvfp4 as Q
from . import nvfp4_train as T
from .lmoe import segments, sqrelu

__all__ = ["experts_backward_nvfp4", "SEEDS"]

SEEDS = {"do": 0, "da": 1, "rht_w2": 2, "do_t": 3, "rht_w1": 4, "da_t": 5}


def _gscale(X: np.ndarray) -> np.float32:
    return np.float32(np.float32(np.max(np.abs(X))) / np.float32(6.0 * 448.0))


def _q_sr(X, seed, on):
    if not on:
        return np.asarray(X, dtype=np.float64)
    return T.fake_quant_sr(np.asarray(X, dtype=np.float32), _gscale(X), seed)


def _q_rn(X, on):
    if not on:
        return np.asarray(X, dtype=np.float64)
    return Q.fake_quant(np.asarray(X, dtype=np.float32), _gscale(X))


def _padded_t(rows: np.ndarray, offsets, counts):
    """[R][f] rows in expert order -> [f][sum of padded counts] with each
    expert's rows at its 16-aligned offset, zeros in the padding."""
    pc = (counts + 15) // 16 * 16
    po = np.concatenate([[0], np.cumsum(pc)])
    out = np.zeros((rows.shape[1], int(po[-1])), dtype=np.float64)
    for e in np.nonzero(counts)[0]:
        out[:, po[e]:po[e] + counts[e]] = rows[offsets[e]:offsets[e + 1]].T
    return out, po


def experts_backward_nvfp4(U: np.ndarray, S: np.ndarray, w: np.ndarray, dv: np.ndarray,
                           get_w1: Callable[[int], np.ndarray], get_w2: Callable[[int], np.ndarray],
                           N: int, g_u: float, g_h: float, seed: int,
                           quant_fwd: bool = True, quant_bwd: bool = True,
                           rht: bool = True) -> Dict[str, object]:
    """Gradients of the routed experts under the NVFP4 recipe.

    U [T][l] latent rows (before quantisation), S [T][K] selected experts,
    w [T][K] router weights, dv [T][l] = dL/dv; get_w1(e) [h][l], get_w2(e)
    [l][h] the BF16 weights; g_u, g_h the forward's static activation scales.
    quant_fwd / quant_bwd / rht switch the forward's quantisation, the
    backward's and the transform off (for the pins).  Returns du [T][l],
    dw [T][K], dW1 / dW2 dicts expert -> [h][l] / [l][h] (every expert some
    token chose), and o [T][K][l] (the forward's expert outputs).
    """
    U = np.asarray(U, dtype=np.float64)
    S = np.asarray(S, dtype=np.int64)
    Tn, K = S.shape
    l = U.shape[1]
    counts, offsets, perm, inv = segments(S, N)
    tok = perm // K
    slot = perm % K
    # forward, rows in expert order
    Uq = Q.fake_quant(U.astype(np.float32), g_u) if quant_fwd else U
    W1q, W2q = {}, {}
    rows_a, rows_g, rows_o = [], [], []
    for e in range(N):
        if counts[e] == 0:
            continue
        w1, w2 = get_w1(e), get_w2(e)
        if quant_fwd:
            w1 = Q.fake_quant(w1, Q.weight_global_scale(w1), block2d=True)
            w2 = Q.fake_quant(w2, Q.weight_global_scale(w2), block2d=True)
        W1q[e], W2q[e] = w1, w2
        r = slice(offsets[e], offsets[e + 1])
        a = Uq[tok[r]] @ w1.T
        g = Q.fake_quant(sqrelu(a), g_h) if quant_fwd else sqrelu(a)
        rows_a.append(a)
        rows_g.append(g)
        rows_o.append(g @ w2.T)
    A = np.concatenate(rows_a)
    G = np.concatenate(rows_g)
    O = np.concatenate(rows_o)
    h = A.shape[1]
    # dL/dw and the output gradient rows
    DV = np.asarray(dv, dtype=np.float64)[tok]
    wr = np.asarray(w, dtype=np.float64)[tok, slot]
    dw = np.zeros((Tn, K))
    dw[tok, slot] = np.sum(DV * O, axis=1)
    DO = wr[:, None] * DV
    # dgrad GEMM2, activation derivative, dgrad GEMM1
    DOq = _q_sr(DO, seed + SEEDS["do"], quant_bwd)
    DG = np.zeros((Tn * K, h))
    for e, w2 in W2q.items():
        r = slice(offsets[e], offsets[e + 1])
        DG[r] = DOq[r] @ w2
    DA = DG * 2.0 * np.maximum(A, 0.0)
    DAq = _q_sr(DA, seed + SEEDS["da"], quant_bwd)
    DUr = np.zeros((Tn * K, l))
    for e, w1 in W1q.items():
        r = slice(offsets[e], offsets[e + 1])
        DUr[r] = DAq[r] @ w1
    du = np.zeros_like(U)
    np.add.at(du, tok, DUr)

    # wgrad GEMMs over each expert's rows, transformed and quantised
    def wgrad(grad_rows, act_rows, s_rht, s_sr):
        Gt, po = _padded_t(grad_rows, offsets, counts)
        At, _ = _padded_t(act_rows, offsets, counts)
        if rht:
            Gt = T.rht16(Gt.astype(np.float32), seed=seed + s_rht).astype(np.float64)
            At = T.rht16(At.astype(np.float32), seed=seed + s_rht).astype(np.float64)
        Gq = _q_sr(Gt, seed + s_sr, quant_bwd)
        Aq = _q_rn(At, quant_bwd)
        out = {}
        for e in np.nonzero(counts)[0]:
            c = slice(po[e], po[e + 1])
            out[int(e)] = Gq[:, c] @ Aq[:, c].T
        return out

    dW2 = wgrad(DO, G, SEEDS["rht_w2"], SEEDS["do_t"])
    dW1 = wgrad(DA, U[tok], SEEDS["rht_w1"], SEEDS["da_t"])
    o = np.zeros((Tn, K, l))
    o[tok, slot] = O
    return {"du": du, "dw": dw, "dW1": dW1, "dW2": dW2, "o": o}
