"""The multi-rank path of bench.py on CPU: two gloo ranks run the timed region
with a host timer, reduce the slowest rank's time and compute whole-job
throughput; each rank draws its own token batch."""
import os
import socket
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        def host_timer():
            t = {}
            return (lambda: t.__setitem__("a", time.perf_counter()),
                    lambda: t.__setitem__("b", time.perf_counter()),
                    lambda: (t["b"] - t["a"]) * 1e3)

        # rank 1 is ten times slower (a margin no scheduler jitter on a busy
        # host closes): the reported time must be its total
        delay = 0.002 if rank == 0 else 0.02
        per_step, total = bench.timed_region(lambda: time.sleep(delay), 5, host_timer)
        own = sum(per_step)
        value = bench.throughput(world, 256, 5, total)
        seed = bench.shard_seed(1, rank)
        from lmoe_synth import CONFIGS, make_weights, make_x
        cfg = CONFIGS["tiny"]
        _, gen = make_weights(cfg, device="cpu")
        g = torch.Generator().manual_seed(seed)
        x = make_x(cfg, g, T=8)
        q.put((rank, own, total, value, seed, x.float().sum().item()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, own0, tot0, val0, seed0, xs0), (r1, own1, tot1, val1, seed1, xs1) = res
    assert tot0 == tot1 == pytest.approx(max(own0, own1))
    assert own1 > own0                      # the slower rank sets the time
    assert val0 == val1 == pytest.approx(world * 256 * 5 / (tot0 / 1e3))
    assert seed0 != seed1 and xs0 != xs1    # each rank has its own batch
