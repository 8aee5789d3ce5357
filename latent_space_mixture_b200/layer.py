"""Python binding of the LatentMoE layer: the C ABI's calls with the same names,
taking torch tensors for device memory and torch streams.  Every step of the
layer runs in the CUDA library; nothing here computes."""
from __future__ import annotations

import ctypes
from ctypes import byref, c_char_p, c_double, c_int64, c_void_p
from typing import Dict, Optional

import torch

from . import _lib
from ._lib import (DBG, FLAG_BACKWARD, FLAG_EP_DENSE, FLAG_NO_PROJECTION, FMT_BF16, FMT_FP8,
                   FMT_NVFP4,
                   FMT_W4A16, NVFP4_WEIGHT_FLAGS,
                   LmoeConfig, LmoeError, LmoeGrads, LmoeWeights, check)

__all__ = ["LatentMoE", "ExpertShard", "lmoe_route", "lmoe_route_status",
           "lmoe_check_bounded_wait", "LmoeError", "lmoe_rht16", "lmoe_nvfp4_quantize_sr",
           "lmoe_permute_rows"]

_WEIGHT_SHAPES = {
    "w_router": ("N", "d"), "w_dn": ("l", "d"), "w1": ("N", "h", "l"), "w2": ("N", "l", "h"),
    "w_upl": ("d", "l"), "w_s1": ("hs", "d"), "w_s2": ("d", "hs"),
}


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


class LatentMoE:
    """lmoe_create / lmoe_forward / lmoe_destroy for one layer.

    weights: dict of CUDA bf16 tensors w_router [N][d], w_dn [l][d],
    w1 [N][h][l], w2 [N][l][h], w_upl [d][l], w_s1 [h_s][d], w_s2 [d][h_s],
    and optionally router_bias [N] fp32.  The library copies them.
    projections=False builds the standard MoE (latent = d, no w_dn / w_upl:
    the experts work on x and their combined output is added as is).
    nvfp4_weights ("1d", "2d", "mse", "2d_mse") picks the NVFP4 weight blocks
    and scale choice (LMOE_FLAG_NVFP4_WEIGHT_* of the C ABI).
    backward=True reserves the workspace of lmoe_backward (LMOE_FLAG_BACKWARD).
    ep_dense=True builds the expert-parallel layer handle (LMOE_FLAG_EP_DENSE):
    no expert weights (w1, w2 not needed), dispatch() and combine() only.
    """

    def __init__(self, d: int, latent: int, n_experts: int, top_k: int, expert_hidden: int,
                 shared_hidden: int, max_tokens: int, weights: Dict[str, torch.Tensor],
                 expert_format: str = "bf16", act_gscales=(0.0, 0.0), projections: bool = True,
                 nvfp4_weights: str = "1d", backward: bool = False, ep_dense: bool = False):
        self.lib = _lib.load()
        dims = {"d": d, "l": latent, "N": n_experts, "h": expert_hidden, "hs": shared_hidden}
        for k, shape in _WEIGHT_SHAPES.items():
            if not projections and k in ("w_dn", "w_upl"):
                continue
            if ep_dense and k in ("w1", "w2"):
                continue
            t = weights[k]
            want = tuple(dims[s] for s in shape)
            if tuple(t.shape) != want or t.dtype != torch.bfloat16 or not t.is_cuda:
                raise ValueError(f"{k}: need CUDA bf16 {want}, got {t.dtype} {tuple(t.shape)}")
            if not t.is_contiguous():
                raise ValueError(f"{k} must be contiguous")
        bias = weights.get("router_bias")
        if bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (n_experts,)
                                 or not bias.is_cuda):
            raise ValueError("router_bias: need CUDA fp32 [N]")
        self.cfg = LmoeConfig(d, latent, n_experts, top_k, expert_hidden, shared_hidden,
                              {"bf16": FMT_BF16, "nvfp4": FMT_NVFP4, "fp8": FMT_FP8,
                               "w4a16": FMT_W4A16}[expert_format],
                              (0 if projections else FLAG_NO_PROJECTION)
                              | NVFP4_WEIGHT_FLAGS[nvfp4_weights]
                              | (FLAG_BACKWARD if backward else 0)
                              | (FLAG_EP_DENSE if ep_dense else 0), max_tokens)
        w = LmoeWeights(weights["w_router"].data_ptr(),
                        bias.data_ptr() if bias is not None else None,
                        weights["w_dn"].data_ptr() if projections else None,
                        None if ep_dense else weights["w1"].data_ptr(),
                        None if ep_dense else weights["w2"].data_ptr(),
                        weights["w_upl"].data_ptr() if projections else None,
                        weights["w_s1"].data_ptr(), weights["w_s2"].data_ptr(),
                        float(act_gscales[0]), float(act_gscales[1]))
        self.device = weights["w_router"].device
        h = c_void_p()
        with torch.cuda.device(self.device):
            check(self.lib.lmoe_create(byref(self.cfg), byref(w), byref(h)), "lmoe_create")
        self.h = h
        self.last_T = 0

    # -- forward ----------------------------------------------------------
    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """lmoe_forward: x [T][d] CUDA bf16 -> y [T][d] CUDA bf16 (async)."""
        if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != self.cfg.d or not x.is_cuda:
            raise ValueError("x: need CUDA bf16 [T][d]")
        x = x.contiguous()
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.cfg.d), dtype=torch.bfloat16, device=x.device)
        check(self.lib.lmoe_forward(self.h, c_void_p(x.data_ptr()), T, c_void_p(out.data_ptr()),
                                    _stream_ptr(stream)), "lmoe_forward")
        self.last_T = T
        return out

    __call__ = forward

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor,
                     stream: Optional[torch.cuda.Stream] = None) -> None:
        """lmoe_forward_host: host (pinned) bf16 buffers in and out, synchronous."""
        if x_host.is_cuda or y_host.is_cuda or x_host.dtype != torch.bfloat16 \
                or y_host.dtype != torch.bfloat16 or x_host.shape != y_host.shape:
            raise ValueError("host bf16 [T][d] buffers required")
        T = x_host.shape[0]
        check(self.lib.lmoe_forward_host(self.h, c_void_p(x_host.data_ptr()), T,
                                         c_void_p(y_host.data_ptr()), _stream_ptr(stream)),
              "lmoe_forward_host")
        self.last_T = T

    # -- expert parallelism -----------------------------------------------
    def dispatch(self, x: torch.Tensor, rows_out: Optional[torch.Tensor] = None,
                 counts_out: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None):
        """lmoe_forward_dispatch: x [T][d] -> (rows [T*K][l] bf16 in expert
        order, counts [N] int32), both on the device (async)."""
        if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != self.cfg.d or not x.is_cuda:
            raise ValueError("x: need CUDA bf16 [T][d]")
        x = x.contiguous()
        T, K = x.shape[0], self.cfg.top_k
        if rows_out is None:
            rows_out = torch.empty((T * K, self.cfg.latent), dtype=torch.bfloat16,
                                   device=x.device)
        if counts_out is None:
            counts_out = torch.empty((self.cfg.n_experts,), dtype=torch.int32, device=x.device)
        check(self.lib.lmoe_forward_dispatch(self.h, c_void_p(x.data_ptr()), T,
                                             c_void_p(rows_out.data_ptr()),
                                             c_void_p(counts_out.data_ptr()),
                                             _stream_ptr(stream)), "lmoe_forward_dispatch")
        self.last_T = T
        return rows_out, counts_out

    def combine(self, rows_in: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """lmoe_forward_combine: the unweighted expert outputs [T*K][l] in the
        last dispatch's row order -> y [T][d] (async)."""
        T = self.last_T
        if rows_in.dtype != torch.bfloat16 or tuple(rows_in.shape) != (T * self.cfg.top_k,
                                                                        self.cfg.latent):
            raise ValueError("rows_in: need bf16 [T*K][l] of the last dispatch")
        rows_in = rows_in.contiguous()
        if out is None:
            out = torch.empty((T, self.cfg.d), dtype=torch.bfloat16, device=rows_in.device)
        check(self.lib.lmoe_forward_combine(self.h, c_void_p(rows_in.data_ptr()), T,
                                            c_void_p(out.data_ptr()), _stream_ptr(stream)),
              "lmoe_forward_combine")
        return out

    # -- backward ---------------------------------------------------------
    GRAD_NAMES = ("d_router", "d_dn", "d_w1", "d_w2", "d_upl", "d_s1", "d_s2")

    def grad_buffers(self) -> Dict[str, torch.Tensor]:
        """Empty fp32 CUDA tensors for every weight gradient, in weight layout."""
        c = self.cfg
        d, l, N, h, hs = c.d, c.latent, c.n_experts, c.expert_hidden, c.shared_hidden
        shapes = {"d_router": (N, d), "d_dn": (l, d), "d_w1": (N, h, l), "d_w2": (N, l, h),
                  "d_upl": (d, l), "d_s1": (hs, d), "d_s2": (d, hs)}
        return {k: torch.empty(v, dtype=torch.float32, device=self.device)
                for k, v in shapes.items()}

    def backward(self, x: torch.Tensor, dy: torch.Tensor, grads: Dict[str, torch.Tensor],
                 dx: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """lmoe_backward of the last forward (x its input): dy [T][d] CUDA bf16
        -> dx [T][d] CUDA bf16; writes the fp32 weight gradients into `grads`
        (tensors from grad_buffers()).  Asynchronous."""
        if dy.dtype != torch.bfloat16 or dy.shape != x.shape or not dy.is_cuda:
            raise ValueError("dy: need CUDA bf16 of x's shape")
        x = x.contiguous()
        dy = dy.contiguous()
        if dx is None:
            dx = torch.empty_like(dy)
        for k in self.GRAD_NAMES:
            t = grads[k]
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{k}: need contiguous CUDA fp32")
        g = LmoeGrads(*[grads[k].data_ptr() for k in self.GRAD_NAMES])
        check(self.lib.lmoe_backward(self.h, c_void_p(x.data_ptr()), c_void_p(dy.data_ptr()),
                                     x.shape[0], c_void_p(dx.data_ptr()), byref(g),
                                     _stream_ptr(stream)), "lmoe_backward")
        return dx

    def experts_backward_nvfp4(self, u: torch.Tensor, topk_idx: torch.Tensor,
                               topk_w: torch.Tensor, dv: torch.Tensor, seed: int,
                               stream: Optional[torch.cuda.Stream] = None
                               ) -> Dict[str, torch.Tensor]:
        """lmoe_experts_backward_nvfp4: the routed experts' forward and
        backward under the NVFP4 training recipe, for u [T][l] bf16, topk_idx
        [T][K] int32, topk_w [T][K] fp32, dv [T][l] bf16 (CUDA).  Returns du
        [T][l] bf16, dw [T][K] fp32, d_w1 [N][h][l] and d_w2 [N][l][h] fp32
        (async)."""
        c = self.cfg
        T = u.shape[0]
        if u.dtype != torch.bfloat16 or dv.dtype != torch.bfloat16 or \
                topk_idx.dtype != torch.int32 or topk_w.dtype != torch.float32:
            raise ValueError("u, dv: bf16 [T][l]; topk_idx int32, topk_w fp32 [T][K]")
        u, dv = u.contiguous(), dv.contiguous()
        topk_idx, topk_w = topk_idx.contiguous(), topk_w.contiguous()
        dev = u.device
        out = {"du": torch.empty((T, c.latent), dtype=torch.bfloat16, device=dev),
               "dw": torch.empty((T, c.top_k), dtype=torch.float32, device=dev),
               "d_w1": torch.empty((c.n_experts, c.expert_hidden, c.latent),
                                   dtype=torch.float32, device=dev),
               "d_w2": torch.empty((c.n_experts, c.latent, c.expert_hidden),
                                   dtype=torch.float32, device=dev)}
        p = lambda t: c_void_p(t.data_ptr())  # noqa: E731
        check(self.lib.lmoe_experts_backward_nvfp4(
            self.h, p(u), p(topk_idx), p(topk_w), p(dv), T, int(seed), p(out["du"]),
            p(out["dw"]), p(out["d_w1"]), p(out["d_w2"]), _stream_ptr(stream)),
            "lmoe_experts_backward_nvfp4")
        self.bw4_T = T
        return out

    def bias_update(self, rate: float = 1e-3, stream: Optional[torch.cuda.Stream] = None) -> None:
        """lmoe_bias_update: aux-loss-free step of the router bias from the
        last forward's expert loads."""
        check(self.lib.lmoe_bias_update(self.h, ctypes.c_float(rate), _stream_ptr(stream)),
              "lmoe_bias_update")

    def sync_status(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        return self.lib.lmoe_sync_status(self.h, _stream_ptr(stream))

    def launches_per_forward(self, T: int) -> int:
        return self.lib.lmoe_launches_per_forward(self.h, int(T))

    # -- debug readout ----------------------------------------------------
    def debug(self, what: str) -> torch.Tensor:
        """lmoe_get_debug: a host copy of an intermediate of the last forward."""
        c, T = self.cfg, self.last_T
        spec = {
            "topk_idx": (torch.int32, (T, c.top_k)), "topk_w": (torch.float32, (T, c.top_k)),
            "counts": (torch.int32, (c.n_experts,)), "offsets": (torch.int32, (c.n_experts + 1,)),
            "perm": (torch.int32, (T * c.top_k,)), "inv": (torch.int32, (T, c.top_k)),
            "logits": (torch.float32, (T, c.n_experts)), "u": (torch.bfloat16, (T, c.latent)),
            "v": (torch.bfloat16, (T, c.latent)), "hs": (torch.bfloat16, (T, c.shared_hidden)),
            "bias": (torch.float32, (c.n_experts,)),
            "scale_tables": (torch.float32, (2, 256)),
            "dv": (torch.bfloat16, (T, c.latent)),
        }
        lp = (c.latent + 255) // 256 * 256
        hp = (c.expert_hidden + 255) // 256 * 256
        N, h, l = c.n_experts, c.expert_hidden, c.latent
        if c.expert_format == FMT_FP8:
            # E4M3 codes, one byte per element, and per-expert scales
            spec.update({"w1q_codes": (torch.uint8, (N * h, l)), "w1q_g": (torch.float32, (N,)),
                         "w2q_codes": (torch.uint8, (N * l, h)), "w2q_g": (torch.float32, (N,))})
        spec.update({} if c.expert_format == FMT_FP8 else {
            "w1q_codes": (torch.uint8, (N * h, lp // 2)),
            "w1q_sf": (torch.uint8, ((N * h // 128) * (lp // 64) * 512,)),
            "w1q_g": (torch.float32, (N,)),
            "w2q_codes": (torch.uint8, (N * l, hp // 2)),
            "w2q_sf": (torch.uint8, ((N * l // 128) * (hp // 64) * 512,)),
            "w2q_g": (torch.float32, (N,)),
        })
        if what.startswith("bw4_"):
            R = getattr(self, "bw4_T", 0) * c.top_k
            C = self.lib.lmoe_nvfp4_bw_columns(self.h)
            spec.update({
                "bw4_do_codes": (torch.uint8, (R, l // 2)), "bw4_do_sf": (torch.uint8, (R, l // 16)),
                "bw4_dot_codes": (torch.uint8, (l, C // 2)), "bw4_dot_sf": (torch.uint8, (l, C // 16)),
                "bw4_ut_codes": (torch.uint8, (l, C // 2)), "bw4_ut_sf": (torch.uint8, (l, C // 16)),
                "bw4_scales": (torch.float32, (16,)), "bw4_seg": (torch.int32, (2, N + 1)),
                "bw4_da": (torch.float32, (R, h))})
        spec = spec[what]
        out = torch.empty(spec[1], dtype=spec[0])
        check(self.lib.lmoe_get_debug(self.h, DBG[what], c_void_p(out.data_ptr()),
                                      out.numel() * out.element_size()), f"debug {what}")
        return out

    # -- profiling --------------------------------------------------------
    def profile_enable(self, on: bool = True) -> None:
        check(self.lib.lmoe_profile_enable(self.h, int(on)), "profile_enable")

    def profile_read(self, reset: bool = True):
        n = 64
        names = (c_char_p * n)()
        ms = (c_double * n)()
        cnt = (c_int64 * n)()
        k = self.lib.lmoe_profile_read(self.h, names, ms, cnt, n, int(reset))
        if k < 0:
            raise LmoeError(k, "profile_read")
        # the forward's kernels always, the backward's when they ran
        return [(names[i].decode(), ms[i], cnt[i]) for i in range(k) if i < 12 or cnt[i] > 0]

    def close(self) -> None:
        if getattr(self, "h", None):
            self.lib.lmoe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ExpertShard:
    """lmoe_experts_create / lmoe_experts_forward: the experts
    [first, first + n_local) of a layer, run on rows handed in by an
    expert-parallel exchange.  w1 [n_local][h][l], w2 [n_local][l][h] CUDA
    bf16 (copied)."""

    def __init__(self, d: int, latent: int, n_experts: int, top_k: int, expert_hidden: int,
                 shared_hidden: int, first: int, w1: torch.Tensor, w2: torch.Tensor,
                 max_rows: int):
        self.lib = _lib.load()
        n = w1.shape[0]
        if w1.dtype != torch.bfloat16 or w2.dtype != torch.bfloat16 or not w1.is_cuda \
                or tuple(w1.shape) != (n, expert_hidden, latent) \
                or tuple(w2.shape) != (n, latent, expert_hidden) \
                or not (w1.is_contiguous() and w2.is_contiguous()):
            raise ValueError("w1 [n][h][l], w2 [n][l][h]: contiguous CUDA bf16")
        self.cfg = LmoeConfig(d, latent, n_experts, top_k, expert_hidden, shared_hidden,
                              FMT_BF16, 0, 1)
        self.first, self.n_local, self.device = first, n, w1.device
        h = c_void_p()
        with torch.cuda.device(self.device):
            check(self.lib.lmoe_experts_create(byref(self.cfg), first, n,
                                               c_void_p(w1.data_ptr()), c_void_p(w2.data_ptr()),
                                               int(max_rows), byref(h)), "lmoe_experts_create")
        self.h = h

    def forward(self, rows: torch.Tensor, counts: torch.Tensor,
                out: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """rows [R][l] bf16 in local expert order, counts [n_local] int32 (both
        CUDA) -> out [R][l] bf16, the unweighted expert outputs (async)."""
        if rows.dtype != torch.bfloat16 or counts.dtype != torch.int32 or not rows.is_cuda:
            raise ValueError("rows: CUDA bf16 [R][l]; counts: CUDA int32 [n_local]")
        rows = rows.contiguous()
        if out is None:
            out = torch.empty_like(rows)
        check(self.lib.lmoe_experts_forward(self.h, c_void_p(rows.data_ptr()),
                                            c_void_p(counts.data_ptr()), rows.shape[0],
                                            c_void_p(out.data_ptr()), _stream_ptr(stream)),
              "lmoe_experts_forward")
        return out

    def sync_status(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        return self.lib.lmoe_sync_status(self.h, _stream_ptr(stream))

    def close(self) -> None:
        if getattr(self, "h", None):
            self.lib.lmoe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lmoe_permute_rows(src: torch.Tensor, idx: torch.Tensor, scatter: bool,
                      out: Optional[torch.Tensor] = None, out_rows: Optional[int] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """lmoe_permute_rows on CUDA row tensors: gather out[r] = src[idx[r]]
    (len(idx) rows out), or scatter out[idx[r]] = src[r] (out_rows rows)."""
    if idx.dtype != torch.int32 or not idx.is_cuda or not src.is_cuda:
        raise ValueError("idx: CUDA int32; src: CUDA")
    src = src.contiguous()
    n = idx.numel()
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else 0
    if out is None:
        rows = (out_rows if out_rows is not None else src.shape[0]) if scatter else n
        out = src.new_empty((rows,) + tuple(src.shape[1:]))
    n_other = out.shape[0] if scatter else src.shape[0]
    if n == 0:
        return out
    check(_lib.load().lmoe_permute_rows(c_void_p(src.data_ptr()), c_void_p(idx.data_ptr()), n,
                                        n_other, row_bytes, c_void_p(out.data_ptr()),
                                        int(scatter), _stream_ptr(stream)), "lmoe_permute_rows")
    return out


def lmoe_route(logits: torch.Tensor, bias: Optional[torch.Tensor], K: int,
               stream: Optional[torch.cuda.Stream] = None) -> Dict[str, torch.Tensor]:
    """lmoe_route: routing and per-expert segments from fp32 logits [T][N]."""
    lib = _lib.load()
    T, N = logits.shape
    dev = logits.device
    logits = logits.contiguous()
    out = {
        "topk_idx": torch.empty((T, K), dtype=torch.int32, device=dev),
        "topk_w": torch.empty((T, K), dtype=torch.float32, device=dev),
        "counts": torch.empty((N,), dtype=torch.int32, device=dev),
        "offsets": torch.empty((N + 1,), dtype=torch.int32, device=dev),
        "perm": torch.empty((T * K,), dtype=torch.int32, device=dev),
        "inv": torch.empty((T, K), dtype=torch.int32, device=dev),
    }
    ws_bytes = lib.lmoe_route_workspace_size(T, N)
    ws = torch.empty((max(ws_bytes, 256),), dtype=torch.uint8, device=dev)
    p = lambda t: c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
    check(lib.lmoe_route(p(logits), p(bias), T, N, K, p(out["topk_idx"]), p(out["topk_w"]),
                         p(out["counts"]), p(out["offsets"]), p(out["perm"]), p(out["inv"]),
                         p(ws), ws.numel(), _stream_ptr(stream)), "lmoe_route")
    out["_workspace"] = ws
    return out


def lmoe_route_status(route_out: Dict[str, torch.Tensor],
                      stream: Optional[torch.cuda.Stream] = None) -> int:
    """lmoe_route_status: waits for the stream and returns the device status
    (0, or the DEVICE code) of the lmoe_route call that produced route_out."""
    T, K = route_out["topk_idx"].shape
    N = route_out["counts"].shape[0]
    ws = route_out["_workspace"]
    return _lib.load().lmoe_route_status(c_void_p(ws.data_ptr()), T, N, _stream_ptr(stream))


def lmoe_rht16(x: torch.Tensor, seed: int, out: Optional[torch.Tensor] = None,
               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """lmoe_rht16: random Hadamard transform of 16-element blocks of fp32
    CUDA rows [rows][cols] (async)."""
    if x.dtype != torch.float32 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x: need CUDA fp32 [rows][cols]")
    x = x.contiguous()
    if out is None:
        out = torch.empty_like(x)
    check(_lib.load().lmoe_rht16(c_void_p(x.data_ptr()), x.shape[0], x.shape[1], int(seed),
                                 c_void_p(out.data_ptr()), _stream_ptr(stream)), "lmoe_rht16")
    return out


def lmoe_nvfp4_quantize_sr(x: torch.Tensor, g: float, seed: int,
                           stream: Optional[torch.cuda.Stream] = None):
    """lmoe_nvfp4_quantize_sr: NVFP4 codes [rows][cols/2] and E4M3 block
    scales [rows][cols/16] of fp32 CUDA rows, elements stochastically rounded
    (async)."""
    if x.dtype != torch.float32 or x.dim() != 2 or not x.is_cuda:
        raise ValueError("x: need CUDA fp32 [rows][cols]")
    x = x.contiguous()
    rows, cols = x.shape
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((rows, cols // 16), dtype=torch.uint8, device=x.device)
    check(_lib.load().lmoe_nvfp4_quantize_sr(c_void_p(x.data_ptr()), rows, cols,
                                             ctypes.c_float(g), int(seed),
                                             c_void_p(codes.data_ptr()),
                                             c_void_p(scales.data_ptr()), _stream_ptr(stream)),
          "lmoe_nvfp4_quantize_sr")
    return codes, scales


def lmoe_check_bounded_wait(limit_ns: int) -> int:
    """lmoe_check_bounded_wait: the status of a wait that nothing completes."""
    return _lib.load().lmoe_check_bounded_wait(int(limit_ns))
