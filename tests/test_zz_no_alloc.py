"""lmoe_route_noalloc, the allocation-free routing entry point, against
lmoe_route (caller-provided workspace) through the C ABI.

Callers that cannot allocate device memory (an engine that reserves all HBM
for its own pool, or a host path where cudaMalloc's implicit device
synchronization is not allowed) use the variant whose scratch is a static
device array.  This file sorts last so that a run stopping at the first
failure has run every other test already; it also passes on its own.
"""
from ctypes import c_void_p

import pytest
import torch

pytestmark = pytest.mark.gpu

W_TOL = 2e-6   # the routing tests' weight tolerance; indices must be equal


def _outputs(T, N, K, dev):
    return {
        "topk_idx": torch.full((T, K), -7, dtype=torch.int32, device=dev),
        "topk_w": torch.full((T, K), -7.0, dtype=torch.float32, device=dev),
        "counts": torch.full((N,), -7, dtype=torch.int32, device=dev),
        "offsets": torch.full((N + 1,), -7, dtype=torch.int32, device=dev),
        "perm": torch.full((T * K,), -7, dtype=torch.int32, device=dev),
        "inv": torch.full((T, K), -7, dtype=torch.int32, device=dev),
    }


def _noalloc(lib, logits, bias, K):
    T, N = logits.shape
    out = _outputs(T, N, K, logits.device)
    p = lambda t: c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
    rc = lib.lmoe_route_noalloc(p(logits), p(bias), T, N, K, p(out["topk_idx"]),
                                p(out["topk_w"]), p(out["counts"]), p(out["offsets"]),
                                p(out["perm"]), p(out["inv"]),
                                c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, out


def test_noalloc_route_matches_workspace_route_two_calls_in_a_row():
    from latent_space_mixture_b200 import _lib, lmoe_route
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    # two calls in a row, the second smaller, so stale scratch would show
    for T, N, K in [(2048, 512, 22), (300, 64, 8)]:
        logits = torch.randn((T, N), generator=g, device=dev) * 1.3
        bias = torch.randn((N,), generator=g, device=dev) * 0.1
        ref = lmoe_route(logits, bias, K)
        torch.cuda.synchronize()
        rc, got = _noalloc(lib, logits, bias, K)
        assert rc == 0
        for k in ("topk_idx", "counts", "offsets", "perm", "inv"):
            assert torch.equal(got[k], ref[k]), k
        assert torch.max(torch.abs(got["topk_w"] - ref["topk_w"])).item() <= W_TOL
        assert lib.lmoe_route_noalloc_status(
            c_void_p(torch.cuda.current_stream().cuda_stream)) == 0


@pytest.mark.parametrize("T,N,K", [(1, 96, 3), (200, 512, 22), (256, 512, 22), (256, 1024, 32),
                                   (33, 32, 32)])
def test_one_block_segments_match_three_kernel_segments(T, N, K):
    """Up to 256 tokens lmoe_route builds the segments in one block (counts
    and chunk bases as popcounts of the chunks' masks in shared memory);
    lmoe_route_noalloc always takes the histogram, scan and scatter kernels.
    Both give the same top-K and bit-identical counts, offsets, perm and inv."""
    from latent_space_mixture_b200 import _lib, lmoe_route
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(13 + T)
    logits = torch.randn((T, N), generator=g, device=dev)
    bias = torch.randn((N,), generator=g, device=dev) * 0.1
    ref = lmoe_route(logits, bias, K)
    torch.cuda.synchronize()
    rc, got = _noalloc(lib, logits, bias, K)
    assert rc == 0
    for k in ("topk_idx", "counts", "offsets", "perm", "inv"):
        assert torch.equal(got[k], ref[k]), k
    assert torch.max(torch.abs(got["topk_w"] - ref["topk_w"])).item() <= W_TOL


def test_noalloc_route_without_bias_and_with_no_tokens():
    from latent_space_mixture_b200 import _lib, lmoe_route
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(12)
    T, N, K = 777, 256, 16
    logits = torch.randn((T, N), generator=g, device=dev)
    ref = lmoe_route(logits, None, K)
    torch.cuda.synchronize()
    rc, got = _noalloc(lib, logits, None, K)
    assert rc == 0
    for k in ("topk_idx", "counts", "offsets", "perm", "inv"):
        assert torch.equal(got[k], ref[k]), k
    assert torch.max(torch.abs(got["topk_w"] - ref["topk_w"])).item() <= W_TOL
    # T = 0: counts and offsets come back zero (the scratch holds the last call's data)
    rc, got = _noalloc(lib, torch.zeros((0, N), device=dev), None, K)
    assert rc == 0
    assert torch.count_nonzero(got["counts"]).item() == 0
    assert torch.count_nonzero(got["offsets"]).item() == 0
    assert lib.lmoe_route_noalloc_status(
        c_void_p(torch.cuda.current_stream().cuda_stream)) == 0


def test_noalloc_route_rejects_sizes_beyond_its_scratch():
    from latent_space_mixture_b200 import _lib
    lib = _lib.load()
    dev = torch.device("cuda", 0)
    logits = torch.zeros((8193, 32), device=dev)
    rc, _ = _noalloc(lib, logits, None, 4)            # T > LMOE_NOALLOC_MAX_TOKENS
    assert rc == -2
    logits = torch.zeros((8192, 64), device=dev)
    rc, _ = _noalloc(lib, logits, None, 33)           # K > 32
    assert rc == -2
