"""The routed experts' backward under the NVFP4 training recipe on the GPU
(lmoe_experts_backward_nvfp4) against the oracle (oracle.backward_nvfp4),
"Nemotron-3 Super 精读报告", section 5.3.

Both sides get the same seeded inputs: latent rows u, the selected experts
and their router weights, dL/dv, the layer's bf16 weights (2D 16 x 16 weight
blocks) and the random-bit seed.

Bit-exact: every quantised tensor whose input both sides compute exactly --
w dv (its codes, E4M3 scales and global scale; stochastic rounding), the
transformed and stochastically rounded (w dv)^T of the W2 weight gradient
and the transformed u^T of the W1 weight gradient (codes in the oracle's
layout, whose expert segments are padded to 16 rows where the GPU pads them
to 256), and the experts' column offsets.

Within a bar: the gradients du, dL/dw, dW1 and dW2, whose inputs pass through
GEMMs (fp32 accumulation against the oracle's float64) before they are
quantised again, so a quantisation boundary can fall between the two sides'
values and move one code by a full step: relative RMS error <= 6e-2, the
NVFP4 layer bar."""
import numpy as np
import pytest
import torch

from lmoe_synth import CONFIGS, act_global_scales, make_weights
from oracle import backward_nvfp4 as B4
from oracle import lmoe as O
from oracle import nvfp4 as Q
from oracle import nvfp4_train as TR

pytestmark = pytest.mark.gpu

TOL = 6e-2
SEED = 1234


def _gscale(X):
    return np.float32(np.float32(np.max(np.abs(X))) / np.float32(2688.0))


def _unpack(codes):
    """packed bytes [..][n/2] (lower index in the low nibble) -> codes [..][n]"""
    c = np.asarray(codes, dtype=np.uint8)
    return np.stack([c & 15, c >> 4], axis=-1).reshape(c.shape[:-1] + (c.shape[-1] * 2,))


def _inputs(cfg, T, seed):
    g = torch.Generator().manual_seed(seed)
    sigma_u = cfg.std * np.sqrt(cfg.d)
    u = (torch.randn((T, cfg.l), generator=g) * sigma_u).to(torch.bfloat16)
    # Zipf-like expert choice, the last two experts never chosen
    pr = torch.tensor([(1.0 + e) ** -1.1 for e in range(cfg.N - 2)] + [0.0, 0.0])
    S = torch.stack([torch.multinomial(pr, cfg.K, replacement=False, generator=g)
                     for _ in range(T)]).to(torch.int32)
    s = torch.rand((T, cfg.K), generator=g) * 0.9 + 0.1
    w = (s / s.sum(dim=1, keepdim=True)).to(torch.float32)
    dv = (torch.randn((T, cfg.l), generator=g) * 0.05).to(torch.bfloat16)
    return u, S, w, dv


def _layer(cfg, w):
    from latent_space_mixture_b200 import LatentMoE
    return LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, 64, w, expert_format="nvfp4",
                     act_gscales=act_global_scales(cfg), nvfp4_weights="2d", backward=True)


def _rms_rel(a, b):
    return float(np.sqrt(np.mean((a - b) ** 2) / max(np.mean(b ** 2), 1e-300)))


@pytest.mark.parametrize("T", [64, 37])
def test_nvfp4_experts_backward_matches_oracle(T):
    cfg = CONFIGS["tiny_nvfp4"].with_(wq="2d")
    w, _ = make_weights(cfg, device="cuda")
    layer = _layer(cfg, w)
    u, S, wt, dv = _inputs(cfg, T, 50 + T)
    out = layer.experts_backward_nvfp4(u.cuda(), S.cuda(), wt.cuda(), dv.cuda(), SEED)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    g_u, g_h = (float(np.float32(x)) for x in act_global_scales(cfg))
    U64, S64 = u.double().numpy(), S.numpy().astype(np.int64)
    w64, dv64 = wt.double().numpy(), dv.double().numpy()
    w1 = lambda e: w["w1"][e].double().cpu().numpy()  # noqa: E731
    w2 = lambda e: w["w2"][e].double().cpu().numpy()  # noqa: E731
    ref = B4.experts_backward_nvfp4(U64, S64, w64, dv64, w1, w2, cfg.N, g_u, g_h, SEED)

    # ---- bit-exact: the quantised tensors of exactly shared inputs --------
    counts, offsets, perm, inv = O.segments(S64, cfg.N)
    tok, slot = perm // cfg.K, perm % cfg.K
    DO = (w64[tok, slot][:, None] * dv64[tok]).astype(np.float32)
    g_do = _gscale(DO)
    codes, sc, _ = TR.quantize_sr(DO, g_do, SEED + B4.SEEDS["do"])
    assert np.array_equal(_unpack(layer.debug("bw4_do_codes").numpy()), codes)
    assert np.array_equal(layer.debug("bw4_do_sf").numpy(), sc)
    scal = layer.debug("bw4_scales").numpy()
    assert scal[8] == g_do

    seg = layer.debug("bw4_seg").numpy()
    DOt, po = B4._padded_t(DO.astype(np.float64), offsets, counts)
    assert np.array_equal(seg[0], po)
    pc = (counts + 15) // 16 * 16
    DOt = TR.rht16(DOt.astype(np.float32), seed=SEED + B4.SEEDS["rht_w2"])
    g_dot = _gscale(DOt)
    dot_codes, dot_sc, _ = TR.quantize_sr(DOt, g_dot, SEED + B4.SEEDS["do_t"])
    Ut, _ = B4._padded_t(U64[tok], offsets, counts)
    Ut = TR.rht16(Ut.astype(np.float32), seed=SEED + B4.SEEDS["rht_w1"])
    g_ut = _gscale(Ut)
    ut_codes, ut_sc, _ = Q.quantize(Ut, g_ut)
    assert scal[10] == g_dot and scal[13] == g_ut
    got_dot = _unpack(layer.debug("bw4_dot_codes").numpy())
    got_dot_sc = layer.debug("bw4_dot_sf").numpy()
    got_ut = _unpack(layer.debug("bw4_ut_codes").numpy())
    got_ut_sc = layer.debug("bw4_ut_sf").numpy()
    for e in np.nonzero(counts)[0]:
        a, b, n = seg[1][e], po[e], pc[e]          # GPU columns, oracle columns, 16-padded rows
        assert np.array_equal(got_dot[:, a:a + n], dot_codes[:, b:b + n]), e
        assert np.array_equal(got_dot_sc[:, a // 16:(a + n) // 16], dot_sc[:, b // 16:(b + n) // 16])
        assert np.array_equal(got_ut[:, a:a + n], ut_codes[:, b:b + n]), e
        assert np.array_equal(got_ut_sc[:, a // 16:(a + n) // 16], ut_sc[:, b // 16:(b + n) // 16])

    # ---- gradients within the NVFP4 bar ----------------------------------
    errs = {"dw": _rms_rel(out["dw"].double().cpu().numpy(), ref["dw"]),
            "du": _rms_rel(out["du"].double().cpu().numpy(), ref["du"])}
    chosen = sorted(ref["dW1"].keys())
    gw1, gw2 = out["d_w1"].cpu().double().numpy(), out["d_w2"].cpu().double().numpy()
    errs["dW1"] = _rms_rel(gw1[chosen], np.stack([ref["dW1"][e] for e in chosen]))
    errs["dW2"] = _rms_rel(gw2[chosen], np.stack([ref["dW2"][e] for e in chosen]))
    unused = sorted(set(range(cfg.N)) - set(chosen))
    assert len(unused) >= 2
    assert not gw1[unused].any() and not gw2[unused].any()
    print("nvfp4 backward T", T, errs)
    for k, v in errs.items():
        assert v <= TOL, (k, v)
    layer.close()


def test_nvfp4_experts_backward_no_rows_and_requirements():
    from latent_space_mixture_b200 import LatentMoE, LmoeError
    cfg = CONFIGS["tiny_nvfp4"].with_(wq="2d")
    w, _ = make_weights(cfg, device="cuda")
    layer = _layer(cfg, w)
    z = torch.zeros((0, cfg.l), dtype=torch.bfloat16, device="cuda")
    out = layer.experts_backward_nvfp4(z, torch.zeros((0, cfg.K), dtype=torch.int32, device="cuda"),
                                       torch.zeros((0, cfg.K), device="cuda"), z, SEED)
    torch.cuda.synchronize()
    assert not out["d_w1"].any() and not out["d_w2"].any()
    layer.close()
    # 1D weight blocks have no transposable scales: no NVFP4 training handle
    with pytest.raises(LmoeError):
        LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, 64, w, expert_format="nvfp4",
                  act_gscales=act_global_scales(cfg), nvfp4_weights="1d", backward=True)


def test_layer_backward_with_nvfp4_experts():
    """lmoe_backward of a layer with 2D-block NVFP4 experts: the routed
    experts under the NVFP4 recipe (seed 0 on the handle's first backward),
    the router, projections and shared expert in BF16.

      * the layer's expert gradients equal, bit for bit, those of
        lmoe_experts_backward_nvfp4 on the layer's own saved u, routing and
        dL/dv (the same kernels on the same values);
      * the saved u and dL/dv against the oracle's X W_dn^T and G W_upl at
        the BF16 bar (relative RMS 1e-2);
      * the oracle's composition of the rest -- the experts' NVFP4 backward
        (oracle.backward_nvfp4) and the router through its dL/dw
        (oracle.backward.router_backward) -- fed the layer's own bf16 u and
        dL/dv and fp32 router weights: the quantised tensors are
        discontinuous in their inputs (a float64 u instead of the bf16 one
        moves a fraction of block scales and stochastic-rounding decisions to
        the neighbouring code, ~0.1 relative RMS on the expert gradients), so
        the oracle starts where the recipe starts.  The gradients through the
        experts within the NVFP4 bar (relative RMS 6e-2), dx, the shared
        expert's and the up-projection's within the BF16 bar (the
        up-projection's from the forward's v, whose u was quantised from the
        fp32 accumulator)."""
    from oracle import backward as B
    from tests._parity import make, to64
    from lmoe_synth import make_grad_out
    cfg = CONFIGS["tiny_nvfp4"].with_(wq="2d")
    w, x, layer = make(cfg, backward=True)
    layer.forward(x)
    dy = make_grad_out(cfg, T=x.shape[0], device="cuda")
    grads = layer.grad_buffers()
    dx = layer.backward(x, dy, grads)
    torch.cuda.synchronize()
    assert layer.sync_status() == 0
    got = {"dx": to64(dx)}
    got.update({k: to64(v) for k, v in grads.items()})
    # the expert part: the entry point on the layer's own inputs
    u, dvg = layer.debug("u"), layer.debug("dv")
    Sg, wg = layer.debug("topk_idx"), layer.debug("topk_w")
    again = layer.experts_backward_nvfp4(u.cuda(), Sg.cuda(), wg.cuda(), dvg.cuda(), 0)
    torch.cuda.synchronize()
    assert np.array_equal(to64(again["d_w1"]), got["d_w1"])
    assert np.array_equal(to64(again["d_w2"]), got["d_w2"])
    # the oracle
    S = Sg.numpy().astype(np.int64)
    X, G = to64(x), to64(dy)
    Wr, b, Wdn, Wupl = to64(w["w_router"]), to64(w["router_bias"]), to64(w["w_dn"]), to64(w["w_upl"])
    Ws1, Ws2 = to64(w["w_s1"]), to64(w["w_s2"])
    S_o, _, gap, s = O.route(X @ Wr.T, b, cfg.K)
    clear = gap > 1e-3
    assert np.array_equal(np.sort(S[clear], 1), np.sort(S_o[clear], 1))
    s_sel = np.take_along_axis(s, S, axis=1)
    wk = s_sel / s_sel.sum(axis=1, keepdims=True)
    U, dv, wl = to64(u), to64(dvg), wg.numpy().astype(np.float64)
    assert _rms_rel(U, X @ Wdn.T) <= 1e-2
    assert _rms_rel(dv, G @ Wupl) <= 1e-2
    assert np.abs(wl - wk).max() <= 1e-5
    g_u, g_h = (float(np.float32(v)) for v in act_global_scales(cfg))
    ref4 = B4.experts_backward_nvfp4(U, S, wl, dv, lambda e: to64(w["w1"][e]),
                                     lambda e: to64(w["w2"][e]), cfg.N, g_u, g_h, 0)
    hs_pre = X @ Ws1.T
    dhs_pre = (G @ Ws2) * 2.0 * np.maximum(hs_pre, 0.0)
    dz = B.router_backward(s_sel, ref4["dw"], S, cfg.N)
    # the forward quantised u from its fp32 accumulator, not from the saved
    # bf16 u: its v against the oracle's forward on the unrounded u
    o_fwd = B4.experts_backward_nvfp4(X @ Wdn.T, S, wk, G @ Wupl, lambda e: to64(w["w1"][e]),
                                      lambda e: to64(w["w2"][e]), cfg.N, g_u, g_h, 0)["o"]
    v = np.einsum("tk,tkl->tl", wk, o_fwd)
    want = {"dx": dhs_pre @ Ws1 + ref4["du"] @ Wdn + dz @ Wr,
            "d_router": dz.T @ X, "d_dn": ref4["du"].T @ X, "d_s1": dhs_pre.T @ X,
            "d_s2": G.T @ O.sqrelu(hs_pre), "d_upl": G.T @ v}
    chosen = sorted(ref4["dW1"].keys())
    errs = {k: _rms_rel(got[k], want[k]) for k in want}
    errs["d_w1"] = _rms_rel(got["d_w1"][chosen], np.stack([ref4["dW1"][e] for e in chosen]))
    errs["d_w2"] = _rms_rel(got["d_w2"][chosen], np.stack([ref4["dW2"][e] for e in chosen]))
    print("nvfp4 layer backward", errs)
    for k in ("dx", "d_s1", "d_s2", "d_upl"):
        assert errs[k] <= 1e-2, (k, errs[k])
    for k in ("d_router", "d_dn", "d_w1", "d_w2"):
        assert errs[k] <= TOL, (k, errs[k])
    layer.close()
