"""Expert parallelism through the library's calls on one GPU: P ranks are
simulated in one process (each with its own dense-only layer handle, its own
tokens and its own shard of experts); the all-to-all of the exchange is done
by device copies along the plan's split sizes (latent_space_mixture_b200.ep
computes the plan; on several GPUs ep.forward runs the same steps with
torch.distributed's all-to-all).  The result must equal the oracle on every
rank's tokens, with the bars of the single-GPU layer.

Exchange volume: one l-wide row per routed (token, expert) pair each way --
the rows LatentMoE narrows from d ("NVIDIA Nemotron 3: Efficient and Open
Intelligence", section 三; "Nemotron-3 Super 精读报告", section 6.5)."""
import numpy as np
import pytest
import torch

from lmoe_synth import CONFIGS, make_weights, make_x
from tests._parity import compare_layer, max_rel, to64

pytestmark = pytest.mark.gpu


def _ranks(cfg, P, T_per):
    from latent_space_mixture_b200 import ExpertShard, LatentMoE, ep
    w, gen = make_weights(cfg, device="cuda")
    x_all = make_x(cfg, gen, T=T_per * P, device="cuda")
    layers, shards = [], []
    for r in range(P):
        lo, hi = ep.expert_range(cfg.N, P, r)
        layers.append(LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, T_per, w,
                                ep_dense=True))
        shards.append(ExpertShard(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, lo,
                                  w["w1"][lo:hi].contiguous(), w["w2"][lo:hi].contiguous(),
                                  max_rows=T_per * P * cfg.K))
    xs = [x_all[r * T_per:(r + 1) * T_per].contiguous() for r in range(P)]
    return w, xs, layers, shards


def _split(t, counts):
    out, a = [], 0
    for c in counts:
        out.append(t[a:a + c])
        a += c
    return out


def _ep_forward(cfg, P, layers, shards, xs):
    """The expert-parallel forward of all P simulated ranks."""
    from latent_space_mixture_b200 import ep, lmoe_permute_rows
    per = cfg.N // P
    sent = [layers[r].dispatch(xs[r]) for r in range(P)]
    counts = torch.stack([c.cpu().to(torch.int64) for _, c in sent])      # [src][N]
    plans = [ep.plan_from_counts(counts[r].reshape(P, per), counts[:, r * per:(r + 1) * per])
             for r in range(P)]
    # all-to-all: rank d receives, source by source, the slice of each
    # source's expert-order rows that belongs to its experts
    pieces = [_split(sent[s][0], plans[s].send_counts) for s in range(P)]
    recv = [torch.cat([pieces[s][d] for s in range(P)]) for d in range(P)]
    back = []
    for d in range(P):
        order = plans[d].local_order.to(torch.int32).cuda()
        local = lmoe_permute_rows(recv[d], order, scatter=False)
        out = shards[d].forward(local, plans[d].local_counts.to(torch.int32).cuda())
        back.append(lmoe_permute_rows(out, order, scatter=True, out_rows=recv[d].shape[0]))
    # reverse all-to-all: each source gets its rows back in the order it sent them
    pieces = [_split(back[d], plans[d].recv_counts) for d in range(P)]
    got = [torch.cat([pieces[d][s] for d in range(P)]) for s in range(P)]
    ys = [layers[r].combine(got[r]) for r in range(P)]
    torch.cuda.synchronize()
    for r in range(P):
        assert layers[r].sync_status() == 0 and shards[r].sync_status() == 0
    return ys, sent, plans


@pytest.mark.parametrize("name,P,T_per", [("tiny", 2, 32), ("tiny", 4, 16), ("tiny", 2, 5),
                                          ("pair_small", 2, 2048)])
def test_expert_parallel_forward_matches_oracle(name, P, T_per):
    """tiny: every token; pair_small: 256-row token blocks in the shards (the
    CTA-pair GEMMs), sampled tokens including each rank's first and last."""
    from latent_space_mixture_b200 import LatentMoE
    cfg = CONFIGS[name]
    w, xs, layers, shards = _ranks(cfg, P, T_per)
    ys, sent, plans = _ep_forward(cfg, P, layers, shards, xs)
    single = LatentMoE(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, T_per, w)
    rng = np.random.default_rng(7)
    for r in range(P):
        # the send buffer is u of each routed row's token, in expert order (exact)
        perm = layers[r].debug("perm").numpy().astype(np.int64)
        u = layers[r].debug("u")
        assert torch.equal(sent[r][0].cpu(), u[torch.from_numpy(perm // cfg.K)])
        assert np.array_equal(sent[r][1].cpu().numpy(), layers[r].debug("counts").numpy())
        T = xs[r].shape[0]
        toks = np.arange(T) if T <= 64 else \
            np.unique(np.concatenate([[0, T - 1], rng.choice(T, 24, replace=False)]))
        errs = compare_layer(layers[r], w, xs[r], ys[r], toks, cfg.K)
        # the single-GPU layer on the same tokens: same kernels, weighting
        # after instead of before the bf16 rounding of the expert outputs;
        # each is within 2e-2 RMS(y) of the oracle, so they are within twice
        # that of each other
        y1 = single.forward(xs[r])
        torch.cuda.synchronize()
        errs["vs_single_gpu_layer"] = max_rel(to64(ys[r]), to64(y1))
        assert errs["vs_single_gpu_layer"] <= 2 * 2e-2
        print(name, P, "rank", r, "rows sent", plans[r].send_counts, errs)
    for o in layers + shards + [single]:
        o.close()


def test_permute_rows_gather_and_scatter_exact():
    from latent_space_mixture_b200 import lmoe_permute_rows
    g = torch.Generator(device="cuda").manual_seed(3)
    src = torch.randn((300, 96), generator=g, device="cuda").to(torch.bfloat16)
    idx = torch.randperm(300, generator=g, device="cuda").to(torch.int32)
    got = lmoe_permute_rows(src, idx, scatter=False)
    assert torch.equal(got, src[idx.long()])
    back = lmoe_permute_rows(got, idx, scatter=True, out_rows=300)
    assert torch.equal(back, src)
    # indices outside the indexed side skip their row
    idx2 = idx.clone()
    idx2[5] = 300
    out = torch.zeros_like(src)
    lmoe_permute_rows(src, idx2, scatter=False, out=out)
    torch.cuda.synchronize()
    assert not out[5].any() and torch.equal(out[6], src[idx[6].long()])


def test_expert_shard_rejects_counts_that_do_not_sum_to_the_rows():
    from latent_space_mixture_b200 import ExpertShard
    cfg = CONFIGS["tiny"]
    w, _ = make_weights(cfg, device="cuda")
    shard = ExpertShard(cfg.d, cfg.l, cfg.N, cfg.K, cfg.h, cfg.hs, 0, w["w1"][:8].contiguous(),
                        w["w2"][:8].contiguous(), max_rows=64)
    rows = torch.randn((40, cfg.l), device="cuda").to(torch.bfloat16)
    out = torch.full_like(rows, 7.0)
    for bad in ([6] * 8, [45, -5, 0, 0, 0, 0, 0, 0]):      # sum 48; a negative count
        counts = torch.tensor(bad, dtype=torch.int32, device="cuda")
        shard.forward(rows, counts, out=out)
        torch.cuda.synchronize()
        assert shard.sync_status() == -6          # DEVICE: nothing computed
        assert torch.all(out == 7.0)
    counts = torch.tensor([5] * 8, dtype=torch.int32, device="cuda")
    shard.forward(rows, counts, out=out)
    torch.cuda.synchronize()
    assert shard.sync_status() == 0
    assert not torch.all(out == 7.0)
    shard.close()
