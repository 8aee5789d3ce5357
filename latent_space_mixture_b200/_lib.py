"""ctypes declarations of the C ABI in include/lmoe.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, Structure, c_char_p, c_double, c_float, c_int, c_int32, c_int64,
                    c_uint64,
                    c_size_t, c_void_p)

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblmoe.so")

LMOE_OK = 0
ERRORS = {-1: "INVALID_ARG", -2: "UNSUPPORTED", -3: "OOM", -4: "CUDA", -5: "TIMEOUT",
          -6: "DEVICE"}
FMT_BF16, FMT_NVFP4, FMT_FP8, FMT_W4A16 = 0, 1, 2, 3
FLAG_NO_PROJECTION = 1   # standard MoE: no latent projections (u = x, r = v)
FLAG_NVFP4_WEIGHT_2D = 2   # NVFP4 weights: one scale per 16 x 16 block
FLAG_NVFP4_WEIGHT_MSE = 4  # NVFP4 weights: MSE-searched block scales
FLAG_BACKWARD = 8   # reserve the workspace of lmoe_backward
FLAG_EP_DENSE = 16  # expert-parallel layer handle without expert weights
NVFP4_WEIGHT_FLAGS = {"1d": 0, "2d": FLAG_NVFP4_WEIGHT_2D, "mse": FLAG_NVFP4_WEIGHT_MSE,
                      "2d_mse": FLAG_NVFP4_WEIGHT_2D | FLAG_NVFP4_WEIGHT_MSE}
DBG = {"topk_idx": 1, "topk_w": 2, "counts": 3, "offsets": 4, "perm": 5, "inv": 6,
       "logits": 7, "u": 8, "v": 9, "hs": 10, "w1q_codes": 11, "w1q_sf": 12, "w1q_g": 13,
       "w2q_codes": 14, "w2q_sf": 15, "w2q_g": 16, "bias": 17,
       "bw4_do_codes": 18, "bw4_do_sf": 19, "bw4_dot_codes": 20, "bw4_dot_sf": 21,
       "bw4_ut_codes": 22, "bw4_ut_sf": 23, "bw4_scales": 24, "bw4_seg": 25, "bw4_da": 26,
       "scale_tables": 27, "dv": 28}


class LmoeConfig(Structure):
    _fields_ = [("d", c_int32), ("latent", c_int32), ("n_experts", c_int32), ("top_k", c_int32),
                ("expert_hidden", c_int32), ("shared_hidden", c_int32),
                ("expert_format", c_int32), ("flags", c_int32), ("max_tokens", c_int64)]


class LmoeWeights(Structure):
    _fields_ = [("w_router", c_void_p), ("router_bias", c_void_p), ("w_dn", c_void_p),
                ("w1", c_void_p), ("w2", c_void_p), ("w_upl", c_void_p), ("w_s1", c_void_p),
                ("w_s2", c_void_p), ("act_gscale_latent", c_float),
                ("act_gscale_hidden", c_float)]


class LmoeGrads(Structure):
    _fields_ = [("d_router", c_void_p), ("d_dn", c_void_p), ("d_w1", c_void_p),
                ("d_w2", c_void_p), ("d_upl", c_void_p), ("d_s1", c_void_p), ("d_s2", c_void_p)]


class LmoeError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        name = ERRORS.get(code, str(code))
        super().__init__(f"lmoe error {name} ({code}){': ' + what if what else ''}")


# exported C symbols with (restype, argtypes)
SIGNATURES = {
    "lmoe_create": (c_int, [POINTER(LmoeConfig), POINTER(LmoeWeights), POINTER(c_void_p)]),
    "lmoe_forward": (c_int, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p]),
    "lmoe_forward_host": (c_int, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p]),
    "lmoe_backward": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_void_p,
                              POINTER(LmoeGrads), c_void_p]),
    "lmoe_bias_update": (c_int, [c_void_p, c_float, c_void_p]),
    "lmoe_sync_status": (c_int, [c_void_p, c_void_p]),
    "lmoe_get_debug": (c_int, [c_void_p, c_int, c_void_p, c_size_t]),
    "lmoe_launches_per_forward": (c_int, [c_void_p, c_int64]),
    "lmoe_profile_enable": (c_int, [c_void_p, c_int]),
    "lmoe_profile_read": (c_int, [c_void_p, POINTER(c_char_p), POINTER(c_double),
                                  POINTER(c_int64), c_int, c_int]),
    "lmoe_route_workspace_size": (c_size_t, [c_int64, c_int32]),
    "lmoe_route": (c_int, [c_void_p, c_void_p, c_int64, c_int32, c_int32, c_void_p, c_void_p,
                           c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                           c_void_p]),
    "lmoe_route_status": (c_int, [c_void_p, c_int64, c_int32, c_void_p]),
    "lmoe_route_noalloc_status": (c_int, [c_void_p]),
    "lmoe_route_noalloc": (c_int, [c_void_p, c_void_p, c_int64, c_int32, c_int32, c_void_p,
                                   c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "lmoe_forward_dispatch": (c_int, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p,
                                      c_void_p]),
    "lmoe_forward_combine": (c_int, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p]),
    "lmoe_experts_create": (c_int, [POINTER(LmoeConfig), c_int32, c_int32, c_void_p, c_void_p,
                                    c_int64, POINTER(c_void_p)]),
    "lmoe_experts_forward": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_void_p,
                                     c_void_p]),
    "lmoe_permute_rows": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int32, c_void_p,
                                  c_int, c_void_p]),
    "lmoe_experts_backward_nvfp4": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_int64, c_uint64, c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_void_p]),
    "lmoe_nvfp4_bw_columns": (c_int64, [c_void_p]),
    "lmoe_nvfp4_quantize": (c_int, [c_void_p, c_int64, c_int32, c_float, c_void_p, c_void_p,
                                    c_void_p]),
    "lmoe_rht16": (c_int, [c_void_p, c_int64, c_int32, c_uint64, c_void_p, c_void_p]),
    "lmoe_nvfp4_quantize_sr": (c_int, [c_void_p, c_int64, c_int32, c_float, c_uint64, c_void_p,
                                       c_void_p, c_void_p]),
    "lmoe_check_bounded_wait": (c_int, [c_int64]),
    "lmoe_destroy": (None, [c_void_p]),
    "lmoe_strerror": (c_char_p, [c_int]),
}

_lib = None


def load() -> ctypes.CDLL:
    """The CUDA library; raises when it has not been built (there is no
    fallback implementation)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m latent_space_mixture_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def check(rc: int, what: str = "") -> None:
    if rc != LMOE_OK:
        raise LmoeError(rc, what)
