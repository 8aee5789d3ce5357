#!/usr/bin/env python
"""Throughput of the LatentMoE layer forward pass on B200 (tokens/s per layer)
and its fraction of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
                    [--impl lmoe|reference]

One step = one lmoe_forward of the workload's T tokens with weights resident
in HBM.  Default workload: the Super-dims decode layer (T=256, d=4096, l=1024,
N=512, K=22, h=2688, h_s=5376, uniform router).  Under torchrun each rank runs
its own token batch (seed + rank) against replicated weights: no collective on
the data path, weak scaling; the timed region is bracketed by barriers and the
reported time is the max over ranks.

At N = 1 the line also carries `workloads`: the Super-dims prefill layer
(T=8192, Zipf router bias), the same with NVFP4 experts, and the Ultra-dims
layer (T=4096), each timed the same way (fewer steps) with its own layer
roofline, dominant-kernel roofline and clock record.

--impl reference times the CPU float64 oracle (the only other implementation
of the layer) on a bounded token sample of the same workload, on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from lmoe_synth import CONFIGS, make_weights, make_x  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "LatentMoE layer tokens/s at 1 B200 (Super dims) and % of roofline"


# ---------------------------------------------------------------------------
# host-side helpers (covered by CPU tests)


def shard_seed(base_seed: int, rank: int) -> int:
    """Token-batch seed of a rank: every rank draws its own batch."""
    return base_seed * 1000 + 17 + rank


def load_peaks(path: str = os.path.join(ROOT, "MEASURED_PEAKS.json")):
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def algorithmic_work(cfg, T: int, counts: np.ndarray):
    """Algorithmic bytes and flops of one forward and of each contraction.

    Bytes count the weights a forward must read (dense weights plus the W1/W2
    of experts with at least one routed row), x and y, and for each kernel its
    own operands and results; flops count real rows only (no tile padding).
    Without projections (the standard MoE) the x-GEMM has no W_dn rows, the
    y-GEMM no W_upl columns, and it reads v once more for the residual add.
    Quantised experts: expert weights and expert inputs at their format's
    bytes per element (NVFP4 0.5 + one E4M3 scale per 16 = 0.5625, FP8 1),
    and the grouped GEMMs' peak is the BF16 peak times the format's nominal
    tensor ratio ("mult": FP4 9/2.25 = 4, FP8 4.5/2.25 = 2).
    """
    d, l, N, K, h, hs = cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs
    lx = l if cfg.proj else 0
    eb = {"bf16": 2.0, "nvfp4": 0.5625, "fp8": 1.0, "w4a16": 0.5625}[cfg.fmt]   # weights
    ea = {"bf16": 2.0, "nvfp4": 0.5625, "fp8": 1.0, "w4a16": 2.0}[cfg.fmt]     # u, H rows
    mult = {"bf16": 1, "nvfp4": 4, "fp8": 2, "w4a16": 1}[cfg.fmt]
    touched = int((counts > 0).sum())
    R = T * K
    wx = (N + lx + hs) * d * 2
    wy = d * (lx + hs) * 2
    wexp = int(touched * h * l * eb)
    per_kernel = {
        "xgemm(router|W_dn|W_s1)": dict(bytes=wx + T * d * 2 + T * (N * 4 + lx * 2 + hs * 2),
                                        flops=2 * T * d * (N + lx + hs)),
        "grouped_gemm1(W1,sqrelu)": dict(bytes=int(wexp + R * l * ea + R * h * ea),
                                         flops=2 * R * l * h, mult=mult),
        "grouped_gemm2(W2,*w)": dict(bytes=int(wexp + R * h * ea + R * l * 2 + R * 4),
                                     flops=2 * R * h * l, mult=mult),
        "ygemm([W_upl|W_s2])": dict(bytes=wy + T * (l + hs) * 2 + T * d * 2,
                                    flops=2 * T * d * (lx + hs)),
    }
    layer = dict(bytes=wx + wy + 2 * wexp + 2 * T * d * 2,
                 flops=sum(v["flops"] for v in per_kernel.values()),
                 # tensor time at the peaks, in units of BF16 flops
                 bf16_equiv_flops=sum(v["flops"] / v.get("mult", 1)
                                      for v in per_kernel.values()))
    return layer, per_kernel


def roofline_entry(name, kw, total_ms, launches, peaks, peak_kind, cfg, T):
    """The roofline object of one kernel from its live CUDA-event times."""
    avg_s = total_ms / 1e3 / max(launches, 1)
    intensity = kw["flops"] / kw["bytes"]
    mult = kw.get("mult", 1)
    p_t = peaks["bf16_tflops"] * mult
    ridge = p_t * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if intensity < ridge:
        achieved = kw["bytes"] / avg_s / 1e9
        return {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None,
                "alg_bytes_per_launch": kw["bytes"], "avg_launch_us": round(avg_s * 1e6, 2),
                "peak_source": peak_kind + " hbm_gbs"}
    achieved = kw["flops"] / avg_s / 1e12
    src = peak_kind + " bf16_tflops (burst)"
    if mult != 1:
        src += f" x {mult} ({'FP4' if mult == 4 else 'FP8'}/BF16 nominal dense ratio)"
    return {"kernel": name, "bound": "tensor", "achieved": round(achieved, 1),
            "peak": round(p_t, 1), "unit": "TFLOP/s",
            "frac": round(achieved / p_t, 4), "traffic": None,
            "alg_flops_per_launch": kw["flops"], "avg_launch_us": round(avg_s * 1e6, 2),
            "peak_source": src}


def measured_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or None
    when there is none or the kernel sources changed since it was taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "roofline_traffic.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return rec.get(workload, {}).get(kernel)
    except (OSError, KeyError, ValueError):
        return None


def max_over_ranks(value: float) -> float:
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
        t = torch.tensor([value], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())
    return value


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def timed_region(step, steps: int, new_timer, between=None):
    """Run `steps` steps bracketed by a barrier on both sides; `new_timer()`
    returns (start, stop, elapsed_ms) callables for one step (CUDA events on
    the GPU); `between()` runs before each step, outside its timer (the L2
    flush).  Returns (per-step ms list, max over ranks of their sum)."""
    timers = [new_timer() for _ in range(steps)]
    barrier()
    for i in range(steps):
        if between is not None:
            between()
        timers[i][0]()
        step()
        timers[i][1]()
    per_step = [t[2]() for t in timers]
    barrier()
    return per_step, max_over_ranks(sum(per_step))


def throughput(world: int, tokens_per_rank: int, steps: int, total_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (total_ms / 1e3)


def cuda_timer(stream):
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)

    def elapsed():
        e.synchronize()
        return s.elapsed_time(e)
    return (lambda: s.record(stream)), (lambda: e.record(stream)), elapsed


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML during a region."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
        self.period = period_s

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, int(rs)))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def stop(self):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self, t0: float, t1: float):
        inside = [s for s in self.samples if t0 <= s[0] <= t1] or self.samples
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = set()
        for _, _, r in inside:
            for name, bit in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for _, m, _ in inside), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(inside)}


def workload_config(cfg, world: int) -> dict:
    """The `config` object of a bench line: the same for both arms."""
    return {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "latent": cfg.l,
            "n_experts": cfg.N, "top_k": cfg.K, "expert_hidden": cfg.h,
            "shared_hidden": cfg.hs, "router_bias": cfg.bias, "expert_format": cfg.fmt,
            "latent_projections": cfg.proj, "tokens_per_rank": cfg.T,
            "parallelism": f"dp{world} (replicated weights)",
            "l2": "256 MiB write between steps, outside the per-step events"}


# ---------------------------------------------------------------------------
# the CPU oracle leg


def oracle_rate(cfg, w, x, seconds: float, seed: int):
    """Tokens/s of the float64 oracle on a bounded sample of the batch, in
    batches of 8 tokens (expert weights fetched and up-cast per expert)."""
    from oracle import lmoe as O

    def to64(t):
        return t.detach().to("cpu").to(torch.float64).numpy()

    dense = {k: (to64(w[k]) if k in w else None)
             for k in ("w_router", "router_bias", "w_dn", "w_upl", "w_s1", "w_s2")}
    rng = np.random.default_rng(seed)
    order = rng.permutation(x.shape[0])
    done, t0 = 0, time.perf_counter()
    while True:
        toks = np.sort(order[done:done + 8])
        if len(toks) == 0:
            break
        xs = to64(x[torch.as_tensor(toks, device=x.device)])
        O.layer_forward(xs, dense["w_router"], dense["router_bias"], dense["w_dn"],
                        lambda e: to64(w["w1"][e]), lambda e: to64(w["w2"][e]), dense["w_upl"],
                        dense["w_s1"], dense["w_s2"], cfg.K)
        done += len(toks)
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count()
    return done / el, done, el, cores


# ---------------------------------------------------------------------------


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="super_decode", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="lmoe", choices=["lmoe", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time the headline workload only (no extra workloads)")
    ap.add_argument("--workload-steps", type=int, default=20,
                    help="timed steps of each extra workload (at most --steps)")
    ap.add_argument("--backward", action="store_true",
                    help="time the training step: forward, backward and the router-bias update")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    cfg = CONFIGS[args.config]

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, cfg, world)

    if args.backward:
        return run_training(args, cfg, world, rank, local_rank)
    return run_forward(args, cfg, world, rank, local_rank)


# Workloads measured beside the headline in the default run (N = 1): the
# other layer sizes and formats the throughput targets name.
EXTRA_WORKLOADS = ("super_prefill", "super_prefill_nvfp4", "ultra")


def make_layer(cfg, T, w):
    from latent_space_mixture_b200 import LatentMoE
    from lmoe_synth import act_global_scales
    return LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, T, w, expert_format=cfg.fmt,
                     act_gscales=act_global_scales(cfg) if cfg.fmt != "bf16" else (0.0, 0.0),
                     projections=cfg.proj, nvfp4_weights=cfg.wq)


def time_forward(layer, x, y, steps, warmup, flush, stream, local_rank):
    """Warm-up, the timed steps (CUDA events per step, L2 flushed between
    them outside the events, clocks sampled meanwhile), then a second pass of
    the same steps with per-kernel events.  Returns (max-over-ranks total ms,
    clock summary, wall seconds of the timed region, per-kernel profile)."""
    for _ in range(warmup):
        layer.forward(x, out=y)
    torch.cuda.synchronize()
    rc = layer.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} after warm-up")
    clocks = ClockSampler(local_rank).start()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    _, total_ms = timed_region(lambda: layer.forward(x, out=y), steps,
                               lambda: cuda_timer(stream), between=flush.zero_)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    clocks.stop()
    # per-kernel times for the roofline: a second pass of the same steps with
    # CUDA events around every kernel (events between kernels serialise them,
    # so this pass is not the headline number)
    layer.profile_enable(True)
    layer.profile_read(reset=True)
    timed_region(lambda: layer.forward(x, out=y), steps, lambda: cuda_timer(stream),
                 between=flush.zero_)
    prof = layer.profile_read(reset=True)
    layer.profile_enable(False)
    rc = layer.sync_status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} after the timed steps")
    return total_ms, clocks.summary(t_wall0, t_wall1), t_wall1 - t_wall0, prof


def forward_rooflines(cfg, T, counts, prof, ms_per_step):
    """The dominant kernel's roofline object, the layer's roofline fractions
    and the per-kernel table of one measured workload."""
    lay, per_kernel = algorithmic_work(cfg, T, counts)
    peaks, peak_kind = load_peaks()
    prof_by = {n: (ms, c) for n, ms, c in prof}
    dom = max((n for n in per_kernel if n in prof_by), key=lambda n: prof_by[n][0])
    roof = roofline_entry(dom, per_kernel[dom], prof_by[dom][0], prof_by[dom][1], peaks,
                          peak_kind, cfg, T)
    roof["traffic"] = measured_traffic(cfg.name, dom)
    kernels = {n: {"ms_total": round(ms, 3), "launches": c,
                   "share": round(ms / max(sum(p[1] for p in prof), 1e-9), 4)}
               for n, ms, c in prof}
    layer_time_s = ms_per_step / 1e3
    layer_roof = {"alg_bytes": lay["bytes"], "alg_flops": lay["flops"],
                  "hbm_frac": round(lay["bytes"] / layer_time_s / 1e9 / peaks["hbm_gbs"], 4),
                  # time roofline: each contraction at its own dtype's peak
                  "tensor_frac": round(lay["bf16_equiv_flops"] / layer_time_s / 1e12
                                       / peaks["bf16_tflops"], 4),
                  "tflops": round(lay["flops"] / layer_time_s / 1e12, 2),
                  "peaks": f"{peak_kind}: HBM {peaks['hbm_gbs']} GB/s, "
                           f"BF16 {peaks['bf16_tflops']} TFLOP/s (burst)"}
    return roof, layer_roof, kernels


def measure_workload(name, args, local_rank, rank, flush, stream):
    """One extra workload on this GPU: its own weights, batch and layer,
    freed before returning."""
    cfg = CONFIGS[name]
    dev = torch.device("cuda", local_rank)
    w, _ = make_weights(cfg, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(shard_seed(cfg.seed, rank))
    x = make_x(cfg, gen, device=dev)
    layer = make_layer(cfg, cfg.T, w)
    del w
    y = torch.empty_like(x)
    steps = max(1, min(args.steps, args.workload_steps))
    total_ms, clk, wall, prof = time_forward(layer, x, y, steps, args.warmup, flush, stream,
                                             local_rank)
    ms = total_ms / steps
    counts = layer.debug("counts").numpy()
    roof, layer_roof, _ = forward_rooflines(cfg, cfg.T, counts, prof, ms)
    out = {"ms_per_step": round(ms, 4), "value": round(throughput(1, cfg.T, steps, total_ms), 1),
           "unit": "tokens/s", "steps": steps, "warmup": args.warmup,
           "config": workload_config(cfg, 1), "layer_roofline": layer_roof, "roofline": roof,
           "clocks": clk, "gpu_launches": layer.launches_per_forward(cfg.T) * steps,
           "wall_s_timed_region": round(wall, 4)}
    layer.close()
    del x, y, layer
    torch.cuda.empty_cache()
    return out


def run_forward(args, cfg, world, rank, local_rank):
    from datetime import timedelta
    torch.cuda.set_device(local_rank)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    from latent_space_mixture_b200 import LatentMoE

    dev = torch.device("cuda", local_rank)
    w, _ = make_weights(cfg, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(shard_seed(cfg.seed, rank))
    x = make_x(cfg, gen, device=dev)
    T = cfg.T
    layer = make_layer(cfg, T, w)
    y = torch.empty_like(x)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > L2
    stream = torch.cuda.current_stream()

    total_ms, clk, wall, prof = time_forward(layer, x, y, args.steps, args.warmup, flush, stream,
                                             local_rank)
    ms_per_step = total_ms / args.steps
    value = throughput(world, T, args.steps, total_ms)
    counts = layer.debug("counts").numpy()
    roof, layer_roof, kernels = forward_rooflines(cfg, T, counts, prof, ms_per_step)

    # end to end through host buffers
    e2e = None
    if not args.no_e2e:
        xh = x.cpu().pin_memory()
        yh = torch.empty_like(xh).pin_memory()
        for _ in range(args.warmup):
            layer.forward_host(xh, yh)
        torch.cuda.synchronize()
        _, e2e_ms = timed_region(lambda: layer.forward_host(xh, yh), args.steps,
                                 lambda: cuda_timer(stream), between=flush.zero_)
        e2e = {"value": round(throughput(world, T, args.steps, e2e_ms), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int(xh.numel() * 2), "d2h_bytes_per_step": int(yh.numel() * 2),
               "ms_per_step": round(e2e_ms / args.steps, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, el, cores = oracle_rate(cfg, w, x, args.cpu_seconds, 1000 + cfg.seed)
        cpu = {"value": round(rate, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} of the {T} tokens of this batch, in batches of 8, {el:.1f} s"}

    # quantised experts (NVFP4, FP8): the quantisation error of the experts'
    # combined output v against the same layer with BF16 experts (GPU against
    # GPU, outside the timed regions), to compare formats and weight recipes
    quant_err = None
    if cfg.fmt != "bf16" and rank == 0:
        v_q = layer.debug("v").float()
        twin = LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, T, w, projections=cfg.proj)
        twin.forward(x, out=torch.empty_like(x))
        torch.cuda.synchronize()
        v_b = twin.debug("v").float()
        twin.close()
        rms = lambda t: float(torch.sqrt(torch.mean(t.double() ** 2)))
        quant_err = {"v_rms_rel_vs_bf16_experts": round(rms(v_q - v_b) / rms(v_b), 5),
                     "format": cfg.fmt}
        if cfg.fmt in ("nvfp4", "w4a16"):
            quant_err["nvfp4_weights"] = cfg.wq

    launches = layer.launches_per_forward(T) * args.steps
    layer.close()
    del w, x, y, layer
    torch.cuda.empty_cache()

    # the other workloads of the throughput targets, one after another on
    # this GPU (N = 1 only: the scaling runs time the headline alone)
    workloads = None
    if world == 1 and not args.no_workloads:
        workloads = {n: measure_workload(n, args, local_rank, rank, flush, stream)
                     for n in EXTRA_WORKLOADS if n != cfg.name}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": DTYPES[cfg.fmt],
            "data": "synthetic (seeded; weights N(0, std) bf16, x N(0,1) bf16)",
            "config": workload_config(cfg, world),
            "roofline": roof, "layer_roofline": layer_roof, "kernels": kernels,
            "kernels_note": "per-kernel CUDA events from a second pass of the same steps",
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk,
            "quantisation_error": quant_err,
            "wall_s_timed_region": round(wall, 4),
            "workloads": workloads,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        torch.distributed.destroy_process_group()
    return 0


DTYPES = {"bf16": "bf16", "nvfp4": "e2m1 experts, bf16 dense", "fp8": "e4m3 experts, bf16 dense",
          "w4a16": "e2m1 weights expanded to f16, f16 activations, bf16 dense"}


TRAIN_METRIC = "LatentMoE layer training step (forward + backward + bias update) tokens/s at 1 B200"


def backward_work(cfg, T: int, counts: np.ndarray):
    """Algorithmic flops and bytes of each backward contraction.  Data
    gradients read the weights (dense ones and the touched experts') and the
    token rows and write the gradient rows; weight gradients read the saved
    activations and the output gradients and write fp32 gradients of every
    weight (all N experts' dW1, dW2).  With NVFP4 experts (the training
    recipe) the experts' GEMMs read 4-bit operands (0.5625 bytes per element
    with their E4M3 block scales), the FC2 data gradient reads the saved bf16
    pre-activation and writes fp32 da."""
    d, l, N, K, h, hs = cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs
    R = T * K
    touched = int((counts > 0).sum())
    wexp = touched * h * l * 2
    if cfg.fmt == "nvfp4":
        q = 0.5625
        wq = int(touched * h * l * q)
        fp4 = {
            "bw dgrad W2^T (dg)": dict(flops=2 * R * l * h,
                                       bytes=wq + int(R * l * q) + R * h * 2 + R * h * 4),
            "bw dgrad W1^T (du rows)": dict(flops=2 * R * h * l,
                                            bytes=wq + int(R * h * q) + R * l * 2),
            "bw wgrad W2": dict(flops=2 * R * l * h, bytes=N * l * h * 4 + int(R * (l + h) * q)),
            "bw wgrad W1": dict(flops=2 * R * h * l, bytes=N * h * l * 4 + int(R * (l + h) * q)),
        }
    else:
        fp4 = {}
    return {
        "bw dgrad [W_upl|W_s2]^T (dv, dhs)": dict(flops=2 * T * d * (l + hs),
                                                  bytes=d * (l + hs) * 2 + T * d * 2 + T * (l + 2 * hs) * 2),
        "bw dgrad W2^T (dg)": dict(flops=2 * R * l * h, bytes=wexp + R * l * 2 + R * h * 2),
        "bw dgrad W1^T (du rows)": dict(flops=2 * R * h * l, bytes=wexp + R * h * 2 + R * l * 2),
        "bw dgrad [W_r;W_dn;W_s1]^T (dx)": dict(flops=2 * T * d * (N + l + hs),
                                                bytes=(N + l + hs) * d * 2 + T * (N + l + hs) * 2
                                                + T * d * 2),
        "bw wgrad [W_upl|W_s2]": dict(flops=2 * T * d * (l + hs),
                                      bytes=d * (l + hs) * 4 + T * (d + l + hs) * 2),
        "bw wgrad W2": dict(flops=2 * R * l * h, bytes=N * l * h * 4 + R * (l + h) * 2),
        "bw wgrad W1": dict(flops=2 * R * h * l, bytes=N * h * l * 4 + R * (l + h) * 2),
        "bw wgrad [W_r;W_dn;W_s1]": dict(flops=2 * T * d * (N + l + hs),
                                         bytes=(N + l + hs) * d * 4 + T * (N + l + hs + d) * 2),
        **fp4,
    }


def oracle_train_rate(cfg, w, x, dy, seconds: float, seed: int):
    """Tokens/s of the float64 oracle's forward + backward on a bounded
    sample of the batch, one token at a time (its expert gradients are
    22 dense matrices per token)."""
    from oracle import backward as OB

    def to64(t):
        return t.detach().to("cpu").to(torch.float64).numpy()

    dense = {k: to64(w[k]) for k in ("w_router", "router_bias", "w_dn", "w_upl", "w_s1", "w_s2")}
    rng = np.random.default_rng(seed)
    order = rng.permutation(x.shape[0])
    done, t0 = 0, time.perf_counter()
    while done < len(order):
        t = int(order[done])
        OB.layer_backward(to64(x[t:t + 1]), dense["w_router"], dense["router_bias"], dense["w_dn"],
                          lambda e: to64(w["w1"][e]), lambda e: to64(w["w2"][e]), dense["w_upl"],
                          dense["w_s1"], dense["w_s2"], cfg.K, to64(dy[t:t + 1]))
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count()
    return done / el, done, el, cores


def run_training(args, cfg, world, rank, local_rank):
    """--backward: one step is lmoe_forward, lmoe_backward and
    lmoe_bias_update on a synthetic batch and upstream gradient (BF16 experts
    with latent projections)."""
    from datetime import timedelta
    torch.cuda.set_device(local_rank)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    from latent_space_mixture_b200 import LatentMoE
    from lmoe_synth import make_grad_out
    if not cfg.proj or not (cfg.fmt == "bf16" or (cfg.fmt == "nvfp4" and "2d" in cfg.wq)):
        raise SystemExit("--backward needs BF16 or 2D-block NVFP4 experts with latent "
                         "projections")
    dev = torch.device("cuda", local_rank)
    w, _ = make_weights(cfg, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(shard_seed(cfg.seed, rank))
    x = make_x(cfg, gen, device=dev)
    T = cfg.T
    dy = make_grad_out(cfg, T=T, device=dev, seed=shard_seed(cfg.seed + 1000, rank))
    from lmoe_synth import act_global_scales
    layer = LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, T, w, expert_format=cfg.fmt,
                      act_gscales=act_global_scales(cfg) if cfg.fmt != "bf16" else (0.0, 0.0),
                      nvfp4_weights=cfg.wq, backward=True)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    grads = layer.grad_buffers()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > L2
    stream = torch.cuda.current_stream()

    def step():
        layer.forward(x, out=y)
        layer.backward(x, dy, grads, dx=dx)
        layer.bias_update(1e-3)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if layer.sync_status() != 0:
        raise RuntimeError("device status after warm-up")
    clocks = ClockSampler(local_rank).start()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    _, total_ms = timed_region(step, args.steps, lambda: cuda_timer(stream), between=flush.zero_)
    torch.cuda.synchronize()
    t_wall1 = time.perf_counter()
    clocks.stop()
    layer.profile_enable(True)
    layer.profile_read(reset=True)
    timed_region(step, args.steps, lambda: cuda_timer(stream), between=flush.zero_)
    prof = layer.profile_read(reset=True)
    layer.profile_enable(False)
    if layer.sync_status() != 0:
        raise RuntimeError("device status after the timed steps")
    ms_per_step = total_ms / args.steps
    value = throughput(world, T, args.steps, total_ms)
    counts = layer.debug("counts").numpy()
    lay, fwd_kernels = algorithmic_work(cfg, T, counts)
    bwd_kernels = backward_work(cfg, T, counts)
    peaks, peak_kind = load_peaks()
    prof_by = {n: (ms, c) for n, ms, c in prof if c > 0}
    dom = max((n for n in bwd_kernels if n in prof_by), key=lambda n: prof_by[n][0])
    roof = roofline_entry(dom, bwd_kernels[dom], prof_by[dom][0], prof_by[dom][1], peaks,
                          peak_kind, cfg, T)
    roof["traffic"] = None
    total_prof = max(sum(v[0] for v in prof_by.values()), 1e-9)
    kernels = {n: {"ms_total": round(ms, 3), "launches": c, "share": round(ms / total_prof, 4)}
               for n, (ms, c) in prof_by.items()}
    step_flops = lay["flops"] + sum(v["flops"] for v in bwd_kernels.values())
    step_roof = {"alg_flops": step_flops,
                 "tflops": round(step_flops / (ms_per_step / 1e3) / 1e12, 2),
                 "tensor_frac": round(step_flops / (ms_per_step / 1e3) / 1e12
                                      / peaks["bf16_tflops"], 4)}

    e2e = None
    if not args.no_e2e:
        xh = x.cpu().pin_memory()
        dyh = dy.cpu().pin_memory()
        dxh = torch.empty_like(xh).pin_memory()
        xd = torch.empty_like(x)
        dyd = torch.empty_like(dy)

        def e2e_step():
            xd.copy_(xh, non_blocking=True)
            dyd.copy_(dyh, non_blocking=True)
            layer.forward(xd, out=y)
            layer.backward(xd, dyd, grads, dx=dx)
            layer.bias_update(1e-3)
            dxh.copy_(dx, non_blocking=True)
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        _, e2e_ms = timed_region(e2e_step, args.steps, lambda: cuda_timer(stream),
                                 between=flush.zero_)
        e2e = {"value": round(throughput(world, T, args.steps, e2e_ms), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int((xh.numel() + dyh.numel()) * 2),
               "d2h_bytes_per_step": int(dxh.numel() * 2),
               "ms_per_step": round(e2e_ms / args.steps, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, el, cores = oracle_train_rate(cfg, w, x, dy, args.cpu_seconds, 1000 + cfg.seed)
        cpu = {"value": round(rate, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} of the {T} tokens (forward + backward, one at a time), {el:.1f} s"}
    # the profiled pass counts every kernel of the library's forward and
    # backward; the bias update adds one
    launches = int(round(sum(c for _, _, c in prof) / args.steps)) + 1
    launches *= args.steps
    if rank == 0:
        line = {
            "metric": TRAIN_METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("bf16 (fp32 accumulation, fp32 weight gradients)" if cfg.fmt == "bf16" else
                      "e2m1 experts (NVFP4 training recipe: fprop, dgrad, wgrad), bf16 dense, "
                      "fp32 weight gradients"),
            "data": "synthetic (seeded; weights N(0, std) bf16, x and dL/dy N(0,1) bf16)",
            "config": {"workload": cfg.name, "T": T, "d": cfg.d, "latent": cfg.l,
                       "n_experts": cfg.N, "top_k": cfg.K, "expert_hidden": cfg.h,
                       "shared_hidden": cfg.hs, "router_bias": cfg.bias,
                       "tokens_per_rank": T, "parallelism": f"dp{world} (replicated weights)",
                       "l2": "256 MiB write between steps, outside the per-step events"},
            "roofline": roof, "step_roofline": step_roof, "kernels": kernels,
            "kernels_note": "per-kernel CUDA events from a second pass of the same steps",
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clocks.summary(t_wall0, t_wall1),
            "wall_s_timed_region": round(t_wall1 - t_wall0, 4),
        }
        print(json.dumps(line), flush=True)
    layer.close()
    if world > 1:
        barrier()
        torch.distributed.destroy_process_group()
    return 0


def run_reference(args, cfg, world):
    """The oracle as the reference arm: each step is the oracle on a bounded
    sample of the workload's tokens (rank 0 only); with --backward, its
    forward + backward."""
    from oracle import lmoe as O  # noqa: F401  (fail early if missing)
    if args.backward and (cfg.fmt != "bf16" or not cfg.proj):
        # the GPU arm's training step has the same restriction
        raise SystemExit("--backward needs a BF16 workload with latent projections")
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w, gen = make_weights(cfg, device=dev)
    x = make_x(cfg, gen, device=dev)
    per_step = max(1.0, 150.0 / max(args.steps + args.warmup, 1))
    if args.backward:
        # the training step's reference: the oracle's forward + backward
        from lmoe_synth import make_grad_out
        dy = make_grad_out(cfg, device=dev)
        rate_fn = lambda sec, seed: oracle_train_rate(cfg, w, x, dy, sec, seed)  # noqa: E731
    else:
        rate_fn = lambda sec, seed: oracle_rate(cfg, w, x, sec, seed)  # noqa: E731
    for _ in range(args.warmup):
        rate_fn(per_step / 4, 7)
    rates, n_tot, el_tot, cores = [], 0, 0.0, 1
    for i in range(args.steps):
        r, n, el, cores = rate_fn(per_step, 1000 + i)
        rates.append(r)
        n_tot += n
        el_tot += el
    value = n_tot / el_tot
    line = {"metric": TRAIN_METRIC if args.backward else METRIC, "value": round(value, 3),
            "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            # a step is the whole workload (T tokens); each timed step ran a
            # bounded sample of it, so this is the sample rate's time for T
            "ms_per_step": round(1e3 * cfg.T / value, 2),
            "sample_ms_per_step": round(1e3 * el_tot / args.steps, 2),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(cfg, world),
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"{n_tot} of the workload's {cfg.T} tokens over "
                                       f"{args.steps} steps, {el_tot:.1f} s"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
