"""Routing and per-expert segments through lmoe_route, bit-exact against the
oracle on logits where the top-K is unique at fp32 precision."""
import numpy as np
import pytest
import torch

from oracle import lmoe as O

pytestmark = pytest.mark.gpu


def _run(logits, bias, K):
    from latent_space_mixture_b200 import lmoe_route
    out = lmoe_route(logits, bias, K)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items() if not k.startswith("_")}


def _separated_logits(T, N, seed):
    """Per token a random permutation of a grid with spacing 1/64 in [-4, 4):
    keys differ by >= 2.8e-4, far above fp32 sigmoid error."""
    g = torch.Generator().manual_seed(seed)
    z = torch.stack([torch.randperm(N, generator=g) for _ in range(T)]).float()
    return (z - N / 2) / (N / 8)


def _check_exact(res, z64, b64, K, N):
    S, w, gap, s = O.route(z64, b64, K)
    assert np.array_equal(res["topk_idx"], S)
    assert np.max(np.abs(res["topk_w"] - w)) <= 2e-6
    counts, offsets, perm, inv = O.segments(S, N)
    assert np.array_equal(res["counts"], counts)
    assert np.array_equal(res["offsets"], offsets)
    assert np.array_equal(res["perm"], perm)
    assert np.array_equal(res["inv"], inv)


@pytest.mark.parametrize("T,N,K", [(1, 32, 4), (31, 64, 8), (33, 512, 22), (1000, 512, 22),
                                   (257, 1024, 32), (64, 32, 32), (300, 96, 1)])
def test_route_exact_on_separated_logits(T, N, K):
    z = _separated_logits(T, N, T * 7 + N)
    res = _run(z.cuda(), None, K)
    _check_exact(res, z.double().numpy(), np.zeros(N), K, N)


def test_route_with_bias_and_empty_experts():
    T, N, K = 500, 128, 6
    z = _separated_logits(T, N, 5)
    b = torch.zeros(N)
    b[:40] = -5.0      # these experts never reach the top-6
    res = _run(z.cuda(), b.cuda(), K)
    _check_exact(res, z.double().numpy(), b.double().numpy(), K, N)
    assert np.all(res["counts"][:40] == 0)


def test_exact_ties_go_to_lower_expert():
    T, N, K = 70, 64, 5
    z = torch.zeros(T, N)
    z[:, 10:20] = 1.0          # ten experts tie for the top
    z[5, 3] = 1.0              # an earlier expert joins the tie for token 5
    res = _run(z.cuda(), None, K)
    S = res["topk_idx"]
    assert np.array_equal(S[0], [10, 11, 12, 13, 14])
    assert np.array_equal(S[5], [3, 10, 11, 12, 13])
    _check_exact(res, z.double().numpy(), np.zeros(N), K, N)
    assert np.allclose(res["topk_w"], 1.0 / K, atol=1e-7)


def test_random_logits_within_gap_window():
    T, N, K = 2048, 512, 22
    g = torch.Generator().manual_seed(3)
    z = torch.randn(T, N, generator=g) * 1.28
    res = _run(z.cuda(), None, K)
    S, w, gap, s = O.route(z.double().numpy(), None, K)
    clear = gap > 1e-5
    assert clear.mean() > 0.9
    assert np.array_equal(np.sort(res["topk_idx"][clear], 1), np.sort(S[clear], 1))
    assert np.allclose(res["topk_w"].sum(1), 1.0, atol=1e-5)


def test_route_status_reads_the_device_record():
    """lmoe_route_status returns OK after a clean call and DEVICE when the
    workspace's error record is set.  The record is the first word of the
    workspace's last 256-byte slot; the test plants a value there on the
    device, since a valid call cannot produce a bad expert index."""
    from latent_space_mixture_b200 import lmoe_route, lmoe_route_status
    T, N, K = 100, 64, 8
    z = _separated_logits(T, N, 9).cuda()
    out = lmoe_route(z, None, K)
    assert lmoe_route_status(out) == 0
    ws = out["_workspace"]
    ws[ws.numel() - 256:ws.numel() - 252] = 1
    assert lmoe_route_status(out) == -6
