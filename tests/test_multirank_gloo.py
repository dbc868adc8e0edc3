"""Data-parallel semantics of dsink on CPU with two gloo ranks.

Each rank owns different sequences of a packed batch.  The sink logit is a
parameter shared by every query of every rank (page "Attention Sink, Learnable
Sink and dsink", section 9: per-rank dsink partials must be combined), so the
sum over ranks of the per-rank dsink must equal dsink of the whole batch; the
other gradients are local.  The oracle stands in for the per-rank compute."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch():
    rng = np.random.default_rng(5)
    lens = [40, 23, 31, 18]
    T, Hq, Hkv, D = sum(lens), 4, 2, 8
    x = {n: rng.standard_normal(s) for n, s in
         (("q", (T, Hq, D)), ("k", (T, Hkv, D)), ("v", (T, Hkv, D)), ("do", (T, Hq, D)))}
    a = rng.standard_normal(Hq)
    return lens, x, a


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    lens, x, a = _batch()
    cu = np.concatenate([[0], np.cumsum(lens)])
    mine = [s for s in range(len(lens)) if s % world == rank]
    rows = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in mine])
    my_cu = np.concatenate([[0], np.cumsum([lens[s] for s in mine])]).astype(np.int32)
    _, _, _, ds = oracle.bwd(x["q"][rows], x["k"][rows], x["v"][rows], a, x["do"][rows], 0.35,
                             causal=True, n_sink=2, window=9, cu_seqlens=my_cu)
    t = torch.from_numpy(ds.copy())
    dist.all_reduce(t)
    out[rank] = t.numpy().tolist()
    dist.barrier()
    dist.destroy_process_group()


def test_dsink_allreduce_over_two_gloo_ranks_equals_full_batch():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    lens, x, a = _batch()
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    _, _, _, full = oracle.bwd(x["q"], x["k"], x["v"], a, x["do"], 0.35, causal=True, n_sink=2,
                               window=9, cu_seqlens=cu)
    for r in range(world):
        np.testing.assert_allclose(np.array(out[r]), full, atol=1e-12)


def _gate_worker(rank, world, port, out):
    """Head importance and the balance-loss gradient under data parallelism
    (page "Attention Sink and the native MoE in attention layers", sections
    4-5: Imp averages the gate over the whole token set): each rank sums its
    gates, the sums and token counts are all-reduced, and every rank feeds
    d loss / d Imp / T_total into its own backward."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    lens, x, a = _batch()
    cu = np.concatenate([[0], np.cumsum(lens)])
    mine = [s for s in range(len(lens)) if s % world == rank]
    rows = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in mine])
    my_cu = np.concatenate([[0], np.cumsum([lens[s] for s in mine])]).astype(np.int32)
    mask = dict(causal=True, n_sink=2, window=9, cu_seqlens=my_cu)
    q, k, v, do = x["q"][rows], x["k"][rows], x["v"][rows], x["do"][rows]
    _, _, ss = oracle.fwd(q, k, v, a, 0.35, **mask)
    acc = torch.from_numpy(np.concatenate([ss.sum(0), [float(len(rows))]]))
    dist.all_reduce(acc)
    acc = acc.numpy()
    imp = acc[:-1] / acc[-1]
    _, d_imp = oracle.gate_aux_loss(imp, lam=0.5, n_shared=1)
    dss = np.broadcast_to(d_imp / acc[-1], ss.shape).copy()
    _, _, _, ds = oracle.bwd(q, k, v, a, do, 0.35, dss=dss, **mask)
    t = torch.from_numpy(ds.copy())
    dist.all_reduce(t)
    out[rank] = (imp.tolist(), t.numpy().tolist())
    dist.barrier()
    dist.destroy_process_group()


def test_gate_statistics_and_gradient_over_two_gloo_ranks_equal_full_batch():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_gate_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    lens, x, a = _batch()
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    mask = dict(causal=True, n_sink=2, window=9, cu_seqlens=cu)
    _, _, ss = oracle.fwd(x["q"], x["k"], x["v"], a, 0.35, **mask)
    imp = oracle.gate_importance(ss)
    _, d_imp = oracle.gate_aux_loss(imp, lam=0.5, n_shared=1)
    dss = np.broadcast_to(d_imp / ss.shape[0], ss.shape).copy()
    _, _, _, full = oracle.bwd(x["q"], x["k"], x["v"], a, x["do"], 0.35, dss=dss, **mask)
    for r in range(world):
        np.testing.assert_allclose(np.array(out[r][0]), imp, atol=1e-14)
        np.testing.assert_allclose(np.array(out[r][1]), full, atol=1e-12)
