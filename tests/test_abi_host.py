"""The C-ABI library on a machine without a GPU: it builds, loads, exports every
entry point include/lmoe.h declares, and rejects bad arguments before any
device work.  No compute calls here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from latent_space_mixture_b200 import build as B
    B.build()
    from latent_space_mixture_b200 import _lib
    return _lib.load()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "lmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lmoe_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("lmoe_create", "lmoe_forward", "lmoe_destroy", "lmoe_get_debug",
              "lmoe_sync_status", "lmoe_strerror", "lmoe_route"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from latent_space_mixture_b200 import _lib
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_strerror(lib):
    assert lib.lmoe_strerror(0) == b"ok"
    assert lib.lmoe_strerror(-5) == b"a bounded device wait ran out"
    assert lib.lmoe_strerror(12345) == b"unknown error"


def _cfg(**kw):
    from latent_space_mixture_b200._lib import LmoeConfig
    base = dict(d=256, latent=64, n_experts=32, top_k=4, expert_hidden=128, shared_hidden=256,
                expert_format=0, flags=0, max_tokens=64)
    base.update(kw)
    return LmoeConfig(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(top_k=33), -1), (dict(top_k=0), -1), (dict(max_tokens=0), -1), (dict(flags=2), -1),
    # no projections: latent must equal d, BF16 experts only
    (dict(flags=1), -2), (dict(flags=1, latent=256, expert_format=1), -2),
    # NVFP4 weight variants need NVFP4 experts; unknown bits are rejected
    (dict(flags=2), -1), (dict(flags=4), -1), (dict(flags=8), -1),
    # FP8 experts: latent and expert hidden multiples of 128
    (dict(expert_format=2), -2), (dict(expert_format=2, flags=2), -1),
    (dict(d=100), -2), (dict(latent=96), -2), (dict(n_experts=48), -2),
    (dict(n_experts=2048, top_k=4), -2), (dict(expert_format=1), -2), (dict(expert_format=7), -1),
])
def test_create_rejects_bad_configs_without_gpu(lib, kw, code):
    from latent_space_mixture_b200._lib import LmoeWeights
    w = LmoeWeights()
    h = ctypes.c_void_p()
    assert lib.lmoe_create(ctypes.byref(_cfg(**kw)), ctypes.byref(w), ctypes.byref(h)) == code
    assert not h.value


def test_null_handle_calls(lib):
    assert lib.lmoe_forward(None, None, 1, None, None) == -1
    assert lib.lmoe_sync_status(None, None) == -1
    assert lib.lmoe_launches_per_forward(None, 1) == -1
    assert lib.lmoe_get_debug(None, 1, None, 0) == -1
    lib.lmoe_destroy(None)


def test_route_argument_checks(lib):
    assert lib.lmoe_route(None, None, 4, 48, 4, *([None] * 6), None, 0, None) == -2   # N % 32
    assert lib.lmoe_route(None, None, 4, 64, 65, *([None] * 6), None, 0, None) == -1  # K > N
    assert lib.lmoe_route(None, None, 4, 64, 8, *([None] * 6), None, 0, None) == -1   # nulls
    assert lib.lmoe_route_workspace_size(1000, 512) >= ((1000 + 31) // 32) * 512 * 4


def test_bounded_wait_limit_checked(lib):
    assert lib.lmoe_check_bounded_wait(10) == -1
    assert lib.lmoe_check_bounded_wait(10**11) == -1
