"""GPU parity at the full benchmark sizes, in the launch configuration bench.py
times (same entry points, shapes and kernels).

The float64 oracle cannot run these problems whole in seconds, so it checks
samples it can compute one by one: forward rows (random plus the first/last
token of every sequence and tile edges), dQ rows, and dK/dV of sampled keys
(from every row that sees them).  dsink, a sum over every query, is checked as
a property at full size: -sum_i Delta_ih exp(a_h - LSE_ih), recomputed in
float64 from the kernels' own O, dO and LSE (the forward rows pin O and LSE).
"""
import numpy as np
import pytest
import torch

import oracle
from learnable_sink_b200 import sinkattn as S
from learnable_sink_b200 import workloads as W

from gpu_util import TOL, check_status, dev, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.clear_status()
    yield
    check_status()


def _boundary_tokens(cu, tile):
    toks = set()
    for a, b in zip(cu[:-1], cu[1:]):
        if b <= a:
            continue
        toks.update([a, b - 1, min(a + tile - 1, b - 1), min(a + tile, b - 1)])
    return sorted(toks)


def _rows(cu, Hq, tile, n_random, rng):
    T = int(cu[-1])
    toks = _boundary_tokens(cu, tile)
    rows = [(t, int(rng.integers(0, Hq))) for t in toks]
    rows += [(int(rng.integers(0, T)), int(rng.integers(0, Hq))) for _ in range(n_random)]
    return np.array(rows, dtype=np.int32)


def _keys(cu, g, tile, n_random, rng):
    T = int(cu[-1])
    toks = _boundary_tokens(cu, tile)
    keys = [(t, g) for t in toks] + [(int(rng.integers(0, T)), g) for _ in range(n_random)]
    return np.array(keys, dtype=np.int32)


def _run_and_check(inp, tile, key_heads, n_rows=160, n_keys=48, seed=0):
    rng = np.random.default_rng(seed)
    T, Hq, Hkv, D = inp.shape
    m = S.Mask.from_spec(inp.mask)
    plan = S.Plan(T, Hq, Hkv, m)
    q, k, v, a, do = (dev(x) for x in (inp.q, inp.k, inp.v, inp.sink, inp.dout))
    out, lse, ss = S.fwd(q, k, v, a, m, plan, scale=inp.scale)
    dq, dk, dv, dsink = S.bwd(q, k, v, out, do, lse, a, m, plan, scale=inp.scale)
    torch.cuda.synchronize()
    tol = TOL[torch.bfloat16]
    kw = inp.mask.oracle_kwargs()
    cu = inp.mask.cu_seqlens.numpy()

    # forward on sampled rows
    rows = _rows(cu, Hq, tile, n_rows, rng)
    ro, rl, rs = oracle.fwd_rows(inp.q, inp.k, inp.v, inp.sink, inp.scale, rows, **kw)
    o = np64(out)[rows[:, 0], rows[:, 1]]
    assert np.abs(o - ro).max() <= tol["o"]
    assert np.abs(np64(lse)[rows[:, 0], rows[:, 1]] - rl).max() <= tol["lse"]
    assert np.abs(np64(ss)[rows[:, 0], rows[:, 1]] - rs).max() <= tol["ss"]

    # backward on sampled rows (dQ) and keys (dK, dV)
    keys = np.concatenate([_keys(cu, g, tile, n_keys // len(key_heads), rng) for g in key_heads])
    sq, sk, sv = oracle.bwd_sampled(inp.q, inp.k, inp.v, inp.sink, inp.dout, inp.scale,
                                    rows, keys, **kw)
    for name, got, ref in (("dq", np64(dq)[rows[:, 0], rows[:, 1]], sq),
                           ("dk", np64(dk)[keys[:, 0], keys[:, 1]], sk),
                           ("dv", np64(dv)[keys[:, 0], keys[:, 1]], sv)):
        err = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30)
        assert err <= tol["grad"], f"{name} relative error {err:.3e}"

    # dsink: sum over every query, recomputed in float64 from O, dO, LSE
    delta = (np64(out) * np64(do)).sum(-1)
    ref_dsink = -(delta * np.exp(inp.sink.double().numpy()[None, :] - np64(lse))).sum(0)
    err = np.abs(np64(dsink) - ref_dsink).max() / np.abs(ref_dsink).max()
    assert err <= 1e-3, f"dsink relative error {err:.3e}"


def test_training_prefill_full_size():
    _run_and_check(W.prefill(), tile=128, key_heads=[0, 5])


def test_streamingllm_band_full_size():
    _run_and_check(W.band(), tile=128, key_heads=[3])


def test_packed_varlen_block_sparse_full_size():
    _run_and_check(W.varlen(), tile=64, key_heads=[6])
