"""Seeded synthetic inputs for the LatentMoE layer (workload configurations).

Shared by the tests, the benchmark and the smoke check to feed both the CUDA
library and the CPU oracle the same values.  Holds no layer arithmetic: only
the configuration table and random draws.

Workloads (dimensions from the pages' layer tables):
  * Super dims: d=4096, l=1024, N=512, K=22, expert hidden 2688, shared hidden
    5376 -- "Nemotron-3 Super 精读报告", table 2.2 (架构配置详表);
  * Ultra dims: d=8192, l=2048, N=512, K=22, expert hidden 5120, shared hidden
    10240 -- "Nemotron 3 Ultra 解读:NVFP4 训出的 Mamba 混合 MoE", section 架构一览;
  * the standard MoE that LatentMoE is compared against: no projections,
    N=128, K=6 at d=4096 with the same expert and shared hidden widths, so
    that total and active expert parameters match Super's 512 x 22 at l=1024
    -- "NVIDIA Nemotron 3: Efficient and Open Intelligence", section 三 eq.(1)
    ("vs 128", "vs 6") and section 六 Table 1.

Draw order per workload (one torch.Generator seeded with the workload's seed,
on the device the tensors are made on): W_r, router-bias permutation, W_dn,
W1 (expert by expert), W2 (expert by expert), W_upl, W_s1, W_s2, x (W_dn and
W_upl are not drawn for a workload without projections).
Weights ~ N(0, std^2) rounded to bf16, x ~ N(0, 1) rounded to bf16.
Router bias: "zero" (uniform router) or "zipf": with a seeded permutation pi
of the experts, rank r_e = 1 + pi(e) and b_e = 0.1 * ln(r_e^-1.1), which makes
per-expert token counts Zipf-like and leaves some experts without tokens.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

__all__ = ["LayerConfig", "CONFIGS", "make_weights", "make_x", "make_grad_out", "act_global_scales"]


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int            # tokens per forward
    d: int            # hidden width
    l: int            # latent width
    N: int            # experts
    K: int            # experts per token
    h: int            # expert hidden width
    hs: int           # shared-expert hidden width
    std: float        # weight init std
    bias: str         # "zero" or "zipf"
    seed: int
    fmt: str = "bf16"  # expert format: "bf16", "nvfp4", "fp8" or "w4a16"
    proj: bool = True  # latent projections W_dn, W_upl (False: standard MoE, l = d)
    wq: str = "1d"     # NVFP4 weight blocks/scales: "1d", "2d", "mse" or "2d_mse"

    def with_(self, **kw) -> "LayerConfig":
        return replace(self, **kw)


CONFIGS: Dict[str, LayerConfig] = {
    # Tiny layer; CPU oracle finishes in seconds
    "tiny": LayerConfig("tiny", 64, 256, 64, 32, 4, 128, 256, 0.02, "zero", 0),
    # Super dims, decode-sized batch: expert weights streamed from HBM
    "super_decode": LayerConfig("super_decode", 256, 4096, 1024, 512, 22, 2688,
                                5376, 0.02, "zero", 1),
    # Super dims, prefill-sized batch, Zipf(1.1) router bias
    "super_prefill": LayerConfig("super_prefill", 8192, 4096, 1024, 512, 22,
                                 2688, 5376, 0.02, "zipf", 2),
    # Ultra dims
    "ultra": LayerConfig("ultra", 4096, 8192, 2048, 512, 22, 5120, 10240,
                         0.015, "zero", 3),
    # Super dims with 64 experts and 32 tokens (11 rows per expert, as in the
    # decode batch): a small case of the same kernels for profiler captures
    "super_decode_n64": LayerConfig("super_decode_n64", 32, 4096, 1024, 64, 22, 2688,
                                    5376, 0.02, "zero", 5),
    # Super dims with 64 experts and 1024 tokens (352 rows per expert, as in
    # the prefill batch), Zipf bias: a small prefill case for profiler captures
    "super_prefill_n64": LayerConfig("super_prefill_n64", 1024, 4096, 1024, 64, 22, 2688,
                                     5376, 0.02, "zipf", 6),
    # mid-sized layer whose token counts reach the CTA-pair GEMMs (256 rows per
    # expert, >= 74 dense 256x256 tiles) at sizes the oracle covers quickly
    "pair_small": LayerConfig("pair_small", 4096, 1024, 512, 64, 4, 512, 1024, 0.03, "zipf", 9),
    # tiny layer with NVFP4 experts (latent and expert hidden multiples of 128)
    "tiny_nvfp4": LayerConfig("tiny_nvfp4", 64, 256, 128, 32, 4, 256, 256, 0.02, "zipf", 7,
                              "nvfp4"),
    # the small prefill case with NVFP4 experts, for profiler captures
    "super_prefill_nvfp4_n64": LayerConfig("super_prefill_nvfp4_n64", 1024, 4096, 1024, 64, 22,
                                           2688, 5376, 0.02, "zipf", 8, "nvfp4"),
    # Super dims decode with NVFP4 experts (weights and activations: W4A4)
    "super_decode_nvfp4": LayerConfig("super_decode_nvfp4", 256, 4096, 1024, 512, 22, 2688, 5376,
                                      0.02, "zero", 1, "nvfp4"),
    # Super dims prefill with NVFP4 experts, Zipf(1.1) router bias
    "super_prefill_nvfp4": LayerConfig("super_prefill_nvfp4", 8192, 4096, 1024,
                                       512, 22, 2688, 5376, 0.02, "zipf", 4,
                                       "nvfp4"),
    # Super prefill with NVFP4 experts whose weights use the pages' other
    # recipes: 2D 16x16 blocks (training) and MSE-searched scales (PTQ)
    # the small prefill case with 2D-block NVFP4 experts: the NVFP4 training
    # backward's kernels at prefill-sized segments, for profiler captures
    "super_prefill_nvfp4_2d_n64": LayerConfig("super_prefill_nvfp4_2d_n64", 1024, 4096, 1024, 64,
                                              22, 2688, 5376, 0.02, "zipf", 8, "nvfp4", wq="2d"),
    "super_prefill_nvfp4_2d": LayerConfig("super_prefill_nvfp4_2d", 8192, 4096, 1024, 512, 22,
                                          2688, 5376, 0.02, "zipf", 4, "nvfp4", wq="2d"),
    "super_prefill_nvfp4_mse": LayerConfig("super_prefill_nvfp4_mse", 8192, 4096, 1024, 512, 22,
                                           2688, 5376, 0.02, "zipf", 4, "nvfp4", wq="mse"),
    # FP8 (E4M3) W8A8 experts: tiny, and Super prefill with Zipf bias
    "tiny_fp8": LayerConfig("tiny_fp8", 64, 256, 128, 32, 4, 256, 256, 0.02, "zipf", 13, "fp8"),
    "super_prefill_fp8": LayerConfig("super_prefill_fp8", 8192, 4096, 1024, 512, 22, 2688, 5376,
                                     0.02, "zipf", 4, "fp8"),
    "super_decode_fp8": LayerConfig("super_decode_fp8", 256, 4096, 1024, 512, 22, 2688, 5376,
                                    0.02, "zero", 1, "fp8"),
    # W4A16 experts (NVFP4 weights, 16-bit activations): tiny, Super decode
    # and prefill ("Nemotron 3 Ultra 解读": one NVFP4 checkpoint serves W4A16)
    "tiny_w4a16": LayerConfig("tiny_w4a16", 64, 256, 128, 32, 4, 256, 256, 0.02, "zipf", 14,
                              "w4a16"),
    "super_decode_w4a16": LayerConfig("super_decode_w4a16", 256, 4096, 1024, 512, 22, 2688, 5376,
                                      0.02, "zero", 1, "w4a16"),
    "super_prefill_w4a16": LayerConfig("super_prefill_w4a16", 8192, 4096, 1024, 512, 22, 2688,
                                       5376, 0.02, "zipf", 4, "w4a16"),
    # the standard-MoE comparator: tiny, decode- and prefill-sized
    "tiny_std": LayerConfig("tiny_std", 64, 256, 256, 32, 4, 128, 256, 0.02, "zipf", 10,
                            proj=False),
    "std_decode": LayerConfig("std_decode", 256, 4096, 4096, 128, 6, 2688, 5376, 0.02,
                              "zero", 11, proj=False),
    "std_prefill": LayerConfig("std_prefill", 8192, 4096, 4096, 128, 6, 2688, 5376, 0.02,
                               "zipf", 12, proj=False),
}


def _randn(shape, std, gen, device):
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
            * std).to(torch.bfloat16)


def make_weights(cfg: LayerConfig, device="cpu", seed: Optional[int] = None):
    """All weights of one layer as bf16 tensors ([out][in] row-major) plus the
    fp32 router bias, drawn in the fixed order of the module docstring.
    Returns (weights dict, generator) -- the generator continues with x."""
    seed = cfg.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    N, d, l, h, hs, sd = cfg.N, cfg.d, cfg.l, cfg.h, cfg.hs, cfg.std
    w = {}
    w["w_router"] = _randn((N, d), sd, gen, device)
    perm = torch.randperm(N, generator=gen, device=device)
    if cfg.bias == "zipf":
        rank = (perm + 1).to(torch.float64)
        w["router_bias"] = (0.1 * (-1.1) * torch.log(rank)).to(torch.float32)
    elif cfg.bias == "zero":
        w["router_bias"] = torch.zeros(N, dtype=torch.float32, device=device)
    else:
        raise ValueError(cfg.bias)
    if cfg.proj:
        w["w_dn"] = _randn((l, d), sd, gen, device)
    elif l != d:
        raise ValueError("a workload without projections has l = d")
    w1 = torch.empty((N, h, l), dtype=torch.bfloat16, device=device)
    for e in range(N):
        w1[e] = _randn((h, l), sd, gen, device)
    w["w1"] = w1
    w2 = torch.empty((N, l, h), dtype=torch.bfloat16, device=device)
    for e in range(N):
        w2[e] = _randn((l, h), sd, gen, device)
    w["w2"] = w2
    if cfg.proj:
        w["w_upl"] = _randn((d, l), sd, gen, device)
    w["w_s1"] = _randn((hs, d), sd, gen, device)
    w["w_s2"] = _randn((d, hs), sd, gen, device)
    return w, gen


def make_x(cfg: LayerConfig, gen: torch.Generator, T: Optional[int] = None,
           device="cpu") -> torch.Tensor:
    """Token batch x [T][d] bf16 ~ N(0, 1), drawn after the weights."""
    T = cfg.T if T is None else T
    return torch.randn((T, cfg.d), generator=gen, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def make_grad_out(cfg: LayerConfig, T: Optional[int] = None, device="cpu",
                  seed: Optional[int] = None) -> torch.Tensor:
    """Upstream gradient dL/dy [T][d] bf16 ~ N(0, 1) for the backward pass,
    from its own generator (seed: the workload's seed + 1000)."""
    T = cfg.T if T is None else T
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed + 1000 if seed is None else seed)
    return torch.randn((T, cfg.d), generator=gen, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def act_global_scales(cfg: LayerConfig):
    """Static scales (u, hidden) of the latent activation u and the expert
    hidden activation for quantised experts, set from the synthetic
    distribution: with sigma_u = std*sqrt(d) and sigma_a = std*sqrt(l)*sigma_u,
    the amax bounds 8*sigma_u and (8*sigma_a)^2 map to E2M1 max (6) times
    E4M3 max (448) for NVFP4 (global scales over E4M3 block scales), or to
    E4M3 max (448) for FP8 (per-tensor scales).  Values beyond the bound
    saturate."""
    sigma_u = cfg.std * math.sqrt(cfg.d)
    sigma_a = cfg.std * math.sqrt(cfg.l) * sigma_u
    top = 448.0 if cfg.fmt == "fp8" else 6.0 * 448.0
    return (8.0 * sigma_u) / top, (8.0 * sigma_a) ** 2 / top
