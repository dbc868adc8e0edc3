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
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    lens, x, a = _batch()
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    _, _, _, full = oracle.bwd(x["q"], x["k"], x["v"], a, x["do"], 0.35, causal=True, n_sink=2,
                               window=9, cu_seqlens=cu)
    for r in range(world):
        np.testing.assert_allclose(np.array(out[r]), full, atol=1e-12)
