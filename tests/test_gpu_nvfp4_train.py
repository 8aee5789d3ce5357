"""GPU parity of the NVFP4 gradient-path pieces (lmoe_rht16,
lmoe_nvfp4_quantize_sr) with the oracle (oracle.nvfp4_train): both sides
compute in float32 in the same order from the same generator, so the
transform's outputs and every code and scale are compared bit-exactly."""
import numpy as np
import pytest
import torch

from oracle import nvfp4 as Q
from oracle import nvfp4_train as T

pytestmark = pytest.mark.gpu


def _inputs(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((rows, cols), generator=g) * torch.exp(torch.randn((rows, 1), generator=g) * 2)
    x[1, 16:32] = 0.0                       # an all-zero block
    x[2, :16] = torch.tensor([0.0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -0.5, 1e9])
    return x.float()


@pytest.mark.parametrize("rows,cols", [(7, 64), (300, 256), (1, 16)])
def test_rht16_bit_exact(rows, cols):
    from latent_space_mixture_b200 import lmoe_rht16
    x = _inputs(max(rows, 3), cols, 1)[:rows]
    for seed in (0, 12345, 2 ** 63 + 7):
        y = lmoe_rht16(x.cuda(), seed).cpu().numpy()
        assert np.array_equal(y.view(np.uint32), T.rht16(x.numpy(), seed=seed).view(np.uint32))


@pytest.mark.parametrize("rows,cols,g", [(7, 64, 0.01), (300, 256, 1e-3), (5, 32, 0.0)])
def test_quantize_sr_bit_exact(rows, cols, g):
    from latent_space_mixture_b200 import lmoe_nvfp4_quantize_sr
    x = _inputs(max(rows, 3), cols, 2)[:rows]
    for seed in (0, 99):
        codes, scales = lmoe_nvfp4_quantize_sr(x.cuda(), g, seed)
        want_c, want_s, _ = T.quantize_sr(x.numpy(), np.float32(g), seed)
        packed = (want_c[:, 0::2] | (want_c[:, 1::2] << 4)).astype(np.uint8)
        assert np.array_equal(scales.cpu().numpy(), want_s)
        assert np.array_equal(codes.cpu().numpy(), packed)


def test_rht_then_sr_is_unbiased_on_the_gpu():
    """The wgrad recipe's composition, averaged over seeds on the GPU,
    recovers the transformed values (SR is unbiased)."""
    from latent_space_mixture_b200 import lmoe_nvfp4_quantize_sr, lmoe_rht16
    x = torch.randn((4, 64), generator=torch.Generator().manual_seed(3)).cuda()
    y = lmoe_rht16(x, 5)
    g = float(y.abs().max()) / (6 * 448)
    acc = np.zeros((4, 64))
    n = 400
    for seed in range(n):
        codes, scales = lmoe_nvfp4_quantize_sr(y, g, 1000 + seed)
        c = codes.cpu().numpy()
        q = np.stack([c & 15, c >> 4], axis=-1).reshape(4, 64)
        sb = Q.e4m3_decode(scales.cpu().numpy()).repeat(16, axis=1)
        acc += Q.e2m1_decode(q) * sb * np.float32(g)
    mean = acc / n
    yv = y.cpu().numpy().astype(np.float64)
    step = Q.e4m3_decode(scales.cpu().numpy()).repeat(16, axis=1) * np.float32(g) * 2.0
    assert np.all(np.abs(mean - yv) <= 5.0 * step / np.sqrt(n) + 1e-12)
