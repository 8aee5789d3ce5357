"""Host-side argument checks of the newer Python entry points (no GPU: they
raise before reaching the library) and the expert-range arithmetic of the
expert-parallel plan."""
import pytest
import torch

from latent_space_mixture_b200 import ep, lmoe_nvfp4_quantize_sr, lmoe_rht16


def test_rht16_and_sr_quantiser_reject_host_tensors():
    x = torch.zeros((2, 32), dtype=torch.float32)
    with pytest.raises(ValueError):
        lmoe_rht16(x, 1)
    with pytest.raises(ValueError):
        lmoe_nvfp4_quantize_sr(x, 0.1, 1)
    with pytest.raises(ValueError):
        lmoe_rht16(torch.zeros(32), 1)


def test_expert_ranges_partition_the_experts():
    N, P = 512, 8
    got = [ep.expert_range(N, P, r) for r in range(P)]
    assert got[0] == (0, 64) and got[-1] == (448, 512)
    assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
    with pytest.raises(ValueError):
        ep.expert_range(10, 4, 0)
