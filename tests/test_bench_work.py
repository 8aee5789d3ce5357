"""Host-side checks of bench.py's algorithmic work model (no GPU)."""
import numpy as np

import bench
from lmoe_synth import CONFIGS


def test_backward_flops_are_twice_the_forward_contractions():
    """Every forward contraction y = W x has two backward ones of the same
    size (dx = W^T dy and dW = dy x^T)."""
    for name in ("tiny", "super_decode", "super_prefill"):
        cfg = CONFIGS[name]
        counts = np.ones(cfg.N, dtype=np.int64)
        fwd, _ = bench.algorithmic_work(cfg, cfg.T, counts)
        bwd = bench.backward_work(cfg, cfg.T, counts)
        assert sum(v["flops"] for v in bwd.values()) == 2 * fwd["flops"]
        assert all(v["bytes"] > 0 for v in bwd.values())


def test_weight_gradient_bytes_cover_fp32_outputs():
    cfg = CONFIGS["super_decode"]
    bwd = bench.backward_work(cfg, cfg.T, np.ones(cfg.N, dtype=np.int64))
    assert bwd["bw wgrad W1"]["bytes"] >= cfg.N * cfg.h * cfg.l * 4
    assert bwd["bw wgrad W2"]["bytes"] >= cfg.N * cfg.h * cfg.l * 4
