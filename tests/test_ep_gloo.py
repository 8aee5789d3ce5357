"""Expert parallelism on CPU: two (and four) gloo ranks, each routing its own
tokens, exchange latent rows with latent_space_mixture_b200.ep, run their
local experts (the oracle's expert FFN stands in for the GPU grouped GEMMs)
and combine; the result equals the single-process oracle on all tokens.
Also: the plan's counts, and a rank whose experts receive no rows."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed, N=8, K=3, d=16, l=8, h=12, hs=10, T=24, bias_scale=0.0):
    """bias_scale < 0: a bias of +5 on the first K experts, which then take
    every token (the other ranks' experts get no rows)."""
    rng = np.random.default_rng(seed)
    b = rng.standard_normal(N) * bias_scale if bias_scale >= 0 else \
        np.where(np.arange(N) < K, 5.0, 0.0)
    p = dict(x=rng.standard_normal((T, d)), W_r=rng.standard_normal((N, d)) * 0.4,
             b=b, W_dn=rng.standard_normal((l, d)) * 0.3,
             W1=rng.standard_normal((N, h, l)) * 0.3, W2=rng.standard_normal((N, l, h)) * 0.3,
             W_upl=rng.standard_normal((d, l)) * 0.3, W_s1=rng.standard_normal((hs, d)) * 0.3,
             W_s2=rng.standard_normal((d, hs)) * 0.3)
    return p, N, K


def _worker(rank, world, port, q, seed, bias_scale):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from latent_space_mixture_b200 import ep
        from oracle import lmoe as O
        p, N, K = _layer(seed, bias_scale=bias_scale)
        T = p["x"].shape[0]
        mine = np.arange(T)[rank::world]                 # this rank's tokens
        x = p["x"][mine]
        z = x @ p["W_r"].T
        S, w, _, _ = O.route(z, p["b"], K)
        counts, offsets, perm, inv = O.segments(S, N)
        u = x @ p["W_dn"].T
        rows = torch.from_numpy(u[perm // K])           # expert-order latent rows
        pl = ep.plan(torch.from_numpy(counts))
        got = ep.dispatch(rows, pl)
        lo, hi = ep.expert_range(N, world, rank)
        # local experts, rows in local expert order
        outs, start = [], 0
        for j, n in enumerate(pl.local_counts.tolist()):
            e = lo + j
            outs.append(O.expert_ffn(got[start:start + n].numpy(), p["W1"][e], p["W2"][e]))
            start += n
        o_local = torch.from_numpy(np.concatenate(outs) if outs else np.zeros((0, u.shape[1])))
        o = ep.combine(o_local, pl).numpy()              # back in this rank's expert order
        v = np.zeros_like(u)
        for t in range(len(mine)):
            for k in range(K):
                v[t] += w[t, k] * o[inv[t, k]]
        y = v @ p["W_upl"].T + O.sqrelu(x @ p["W_s1"].T) @ p["W_s2"].T
        q.put((rank, mine, y, list(pl.send_counts), list(pl.recv_counts),
               pl.local_counts.tolist(), counts.tolist()))
    finally:
        dist.destroy_process_group()


def _bw_worker(rank, world, port, q, seed):
    """Forward and backward with expert parallelism: the output-gradient rows
    take the forward's plan to the experts' owners (dispatch), the latent
    input gradients come back by combine; each rank keeps its experts'
    weight gradients."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from latent_space_mixture_b200 import ep
        from oracle import lmoe as O
        p, N, K = _layer(seed)
        T = p["x"].shape[0]
        G = np.random.default_rng(seed + 7).standard_normal((T, p["x"].shape[1]))
        mine = np.arange(T)[rank::world]
        x = p["x"][mine]
        S, w, _, _ = O.route(x @ p["W_r"].T, p["b"], K)
        counts, offsets, perm, inv = O.segments(S, N)
        tok, slot = perm // K, perm % K
        u = x @ p["W_dn"].T
        pl = ep.plan(torch.from_numpy(counts))
        u_loc = ep.dispatch(torch.from_numpy(u[tok]), pl).numpy()
        lo, _ = ep.expert_range(N, world, rank)
        seg = np.concatenate([[0], np.cumsum(pl.local_counts.numpy())])
        o_loc = np.zeros_like(u_loc)
        for j in range(N // world):
            r = slice(seg[j], seg[j + 1])
            o_loc[r] = O.expert_ffn(u_loc[r], p["W1"][lo + j], p["W2"][lo + j])
        o = ep.combine(torch.from_numpy(o_loc), pl).numpy()      # sender's expert order
        # backward: dv at this rank, the expert-side gradients at the owners
        dv = G[mine] @ p["W_upl"]
        do = w[tok, slot][:, None] * dv[tok]
        do_loc = ep.dispatch(torch.from_numpy(do), pl).numpy()
        du_loc = np.zeros_like(u_loc)
        dW1, dW2 = {}, {}
        for j in range(N // world):
            e, r = lo + j, slice(seg[j], seg[j + 1])
            a = u_loc[r] @ p["W1"][e].T
            g = O.sqrelu(a)
            dW2[e] = do_loc[r].T @ g
            da = (do_loc[r] @ p["W2"][e]) * 2.0 * np.maximum(a, 0.0)
            dW1[e] = da.T @ u_loc[r]
            du_loc[r] = da @ p["W1"][e]
        du_rows = ep.combine(torch.from_numpy(du_loc), pl).numpy()
        du = np.zeros_like(u)
        np.add.at(du, tok, du_rows)
        dw = np.zeros((len(mine), K))
        dw[tok, slot] = np.sum(dv[tok] * o, axis=1)
        q.put((rank, mine, du, dw, dW1, dW2))
    finally:
        dist.destroy_process_group()


def test_ep_backward_matches_single_process():
    from oracle import backward as B
    world, seed = 2, 5
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bw_worker, args=(r, world, port, q, seed))
             for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda r: r[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p, N, K = _layer(seed)
    G = np.random.default_rng(seed + 7).standard_normal((p["x"].shape[0], p["x"].shape[1]))
    ref = B.layer_backward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: p["W1"][e],
                           lambda e: p["W2"][e], p["W_upl"], p["W_s1"], p["W_s2"], K, G)
    seen = set()
    for rank, mine, du, dw, dW1, dW2 in res:
        np.testing.assert_allclose(du, ref["du"][mine], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dw, ref["dw"][mine], rtol=0, atol=1e-12)
        for e in dW1:
            if e in ref["dW1"]:
                np.testing.assert_allclose(dW1[e], ref["dW1"][e], rtol=0, atol=1e-12)
                np.testing.assert_allclose(dW2[e], ref["dW2"][e], rtol=0, atol=1e-12)
            else:
                assert not dW1[e].any() and not dW2[e].any()
            seen.add(e)
    assert seen == set(range(N))


def _run(world, seed, bias_scale=0.0):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, seed, bias_scale))
             for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda r: r[0])
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    return res


def _check(world, seed, bias_scale=0.0):
    from oracle import lmoe as O
    res = _run(world, seed, bias_scale)
    p, N, K = _layer(seed, bias_scale=bias_scale)
    ref = O.layer_forward(p["x"], p["W_r"], p["b"], p["W_dn"], lambda e: p["W1"][e],
                          lambda e: p["W2"][e], p["W_upl"], p["W_s1"], p["W_s2"], K)
    per = N // world
    all_counts = np.array([r[6] for r in res])          # [rank][expert]
    for rank, mine, y, send, recv, local, counts in res:
        np.testing.assert_allclose(y, ref["y"][mine], rtol=0, atol=1e-12)
        # what a rank sends to d is its rows of d's experts; what it gets from
        # s is s's rows of its own experts
        assert send == [int(sum(counts[d * per:(d + 1) * per])) for d in range(world)]
        assert recv == [int(all_counts[s, rank * per:(rank + 1) * per].sum()) for s in range(world)]
        assert local == all_counts[:, rank * per:(rank + 1) * per].sum(axis=0).tolist()
    return all_counts


def test_ep_two_ranks_matches_single_process():
    _check(2, seed=0)


def test_ep_four_ranks_matches_single_process():
    _check(4, seed=1)


def test_ep_rank_without_rows():
    """Every token picks the first K experts (all on rank 0): rank 1 receives
    no rows and runs no expert, the exchange still completes and matches."""
    counts = _check(2, seed=2, bias_scale=-1.0)
    assert counts[:, 4:].sum() == 0 and counts[:, :3].sum() == 2 * 12 * 3


def test_ep_with_router_bias():
    _check(2, seed=4, bias_scale=0.3)
