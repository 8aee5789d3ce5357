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


def test_nvfp4_backward_bytes_count_four_bit_operands():
    """With NVFP4 experts the experts' backward GEMMs read 4-bit operands
    (0.5625 bytes per element with their block scales) and still write fp32
    weight gradients; their flops are those of the BF16 layer."""
    bf, fp = CONFIGS["super_prefill"], CONFIGS["super_prefill_nvfp4_2d"]
    counts = np.ones(bf.N, dtype=np.int64)
    b16 = bench.backward_work(bf, bf.T, counts)
    b4 = bench.backward_work(fp, fp.T, counts)
    R = fp.T * fp.K
    for k in ("bw wgrad W1", "bw wgrad W2"):
        assert b4[k]["flops"] == b16[k]["flops"]
        assert b4[k]["bytes"] == fp.N * fp.h * fp.l * 4 + int(R * (fp.l + fp.h) * 0.5625)
        assert b4[k]["bytes"] < b16[k]["bytes"]
    for k in ("bw dgrad W2^T (dg)", "bw dgrad W1^T (du rows)"):
        assert b4[k]["flops"] == b16[k]["flops"]


def _reference_line(monkeypatch, capsys, name, backward=False):
    import argparse
    import json
    monkeypatch.setattr(bench, "oracle_rate", lambda cfg, w, x, sec, seed: (4.0, 8, 2.0, 3))
    monkeypatch.setattr(bench, "oracle_train_rate",
                        lambda cfg, w, x, dy, sec, seed: (1.0, 2, 2.0, 3))
    args = argparse.Namespace(steps=2, warmup=3, backward=backward)
    bench.run_reference(args, CONFIGS[name], 1)
    return json.loads(capsys.readouterr().out.strip().splitlines()[-1])


def test_reference_arm_reports_the_gpu_arms_config_and_a_full_step(monkeypatch, capsys):
    """The reference line names the same config as the GPU line, and its
    ms_per_step is the time of one whole step (T tokens) at its rate."""
    cfg = CONFIGS["tiny"]
    line = _reference_line(monkeypatch, capsys, "tiny")
    assert line["config"] == bench.workload_config(cfg, 1)
    assert line["impl"] == "reference"
    assert line["value"] == 4.0
    assert abs(line["ms_per_step"] - 1e3 * cfg.T / 4.0) < 1e-6


def test_reference_training_arm_refuses_what_the_gpu_arm_refuses(monkeypatch, capsys):
    import pytest
    with pytest.raises(SystemExit):
        _reference_line(monkeypatch, capsys, "tiny_std", backward=True)
    with pytest.raises(SystemExit):
        _reference_line(monkeypatch, capsys, "tiny_fp8", backward=True)
