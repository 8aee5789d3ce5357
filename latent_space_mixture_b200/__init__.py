"""B200-native (sm_100a) LatentMoE layer: forward pass, backward pass with the
aux-loss-free router-bias update, and the expert-parallel exchange plan.

The layer (NVIDIA Nemotron 3): a sigmoid router with expert biasing at hidden
width d picks the top-K experts and renormalises their weights; a BF16
down-projection maps tokens to the latent width l, where the experts
(squared-ReLU FFNs) run; their weighted sum is projected back to d and added
to a d-wide shared expert.

All of the layer's arithmetic runs in liblmoe.so (hand-written CUDA for
sm_100a behind the C ABI of include/lmoe.h).  This package only marshals
arguments: every entry point loads the library first and raises when it has
not been built (there is no other implementation to fall back to); `ep`
plans the expert-parallel exchange and moves rows with torch.distributed.
"""
from . import ep
from ._lib import LmoeError
from .layer import (ExpertShard, LatentMoE, lmoe_check_bounded_wait, lmoe_nvfp4_quantize_sr,
                    lmoe_permute_rows, lmoe_rht16, lmoe_route, lmoe_route_status)

__all__ = ["LatentMoE", "ExpertShard", "lmoe_permute_rows", "lmoe_route", "lmoe_route_status", "lmoe_check_bounded_wait", "LmoeError", "lmoe_rht16",
           "lmoe_nvfp4_quantize_sr", "ep"]
