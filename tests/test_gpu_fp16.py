"""The f16 element type (SINKATTN_FP16) on the tensor-core path: forward,
backward, decode and the sink-free gate against the float64 oracle, on seeded
inputs generated as for the bf16 cases and rounded to f16.  The kernels are
the bf16 ones with the MMA operand format, the rounding of P / dS / outputs
and the widening of pairs switched to f16."""
import numpy as np
import pytest
import torch

import oracle
from learnable_sink_b200 import sinkattn as S
from learnable_sink_b200 import workloads as W

from gpu_util import TOL, check_lse, check_status, dev, max_abs, np64, rel_err, run_bwd, run_fwd

pytestmark = pytest.mark.gpu

F16 = torch.float16


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.clear_status()
    yield
    check_status()


def _spec(cu, causal=True, n_sink=0, window=0):
    return W.MaskSpec(causal=causal, n_sink=n_sink, window=window,
                      cu_seqlens=torch.tensor(cu, dtype=torch.int32))


def _check_fwd(inp, out, lse, ss):
    tol = TOL[F16]
    assert out.dtype == F16
    ro, rl, rs = oracle.fwd(inp.q, inp.k, inp.v, inp.sink, inp.scale, **inp.mask.oracle_kwargs())
    eo = max_abs(np64(out), ro)
    assert eo <= tol["o"], f"O max abs {eo:.3e}"
    check_lse(np64(lse), rl, tol["lse"])
    assert max_abs(np64(ss), rs) <= tol["ss"]


def _check_bwd(inp, grads):
    tol = TOL[F16]
    dq, dk, dv, dsink = grads
    r = oracle.bwd(inp.q, inp.k, inp.v, inp.sink, inp.dout, inp.scale, **inp.mask.oracle_kwargs())
    for name, got, ref in (("dq", dq, r[0]), ("dk", dk, r[1]), ("dv", dv, r[2])):
        assert got.dtype == F16
        e = rel_err(np64(got), ref)
        assert e <= tol["grad"], f"{name} rel {e:.3e}"
    if inp.sink is not None:
        e = rel_err(np64(dsink), r[3])
        assert e <= tol["grad"], f"dsink rel {e:.3e}"


CASES = {
    "causal_ragged_D128_G4": dict(cu=[0, 300, 555], Hq=8, Hkv=2, D=128),
    "causal_D64_G4": dict(cu=[0, 384], Hq=8, Hkv=2, D=64),
    "band_D128": dict(cu=[0, 900], Hq=4, Hkv=2, D=128, n_sink=4, window=200),
    "band_varlen_D64_G2": dict(cu=[0, 50, 700], Hq=4, Hkv=2, D=64, n_sink=4, window=130),
    # reverse lists long enough to be split: fp32 dK/dV accumulators
    "causal_split_list_D128": dict(cu=[0, 4300], Hq=4, Hkv=1, D=128),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fp16_forward_backward(name):
    cfg = dict(CASES[name])
    cu = cfg.pop("cu")
    mask = _spec(cu, n_sink=cfg.pop("n_sink", 0), window=cfg.pop("window", 0))
    inp = W.make_attn(name, T_tot=cu[-1], dtype=F16, mask=mask, seed=41, **cfg)
    out, lse, ss, m, plan = run_fwd(inp)
    _check_fwd(inp, out, lse, ss)
    _check_bwd(inp, run_bwd(inp, out, lse, m, plan))


@pytest.mark.parametrize("G,D,block", [(8, 64, 64), (4, 128, 64), (4, 128, 128)])
def test_fp16_block_sparse(G, D, block):
    cu = W.random_cu_seqlens(1400, 100, 600, 43)
    bi = W.random_block_indices(cu, 2, block, block, 4, 44, shuffle=True)
    mask = W.MaskSpec(causal=True, cu_seqlens=cu, block_indices=bi, block_q=block, block_k=block)
    inp = W.make_attn("bs_f16", T_tot=int(cu[-1]), Hq=2 * G, Hkv=2, D=D, dtype=F16, mask=mask,
                      seed=45)
    out, lse, ss, m, plan = run_fwd(inp)
    _check_fwd(inp, out, lse, ss)
    _check_bwd(inp, run_bwd(inp, out, lse, m, plan))


@pytest.mark.parametrize("G,D,splits", [(4, 128, 0), (8, 64, 3), (1, 128, 7)])
def test_fp16_decode(G, D, splits):
    d = W.decode(B=6, n_sink=4, window=60, Hq=2 * G, Hkv=2, D=D, dtype=F16, seqlen_range=(0, 100))
    d.cache_seqlens = torch.tensor([0, 1, 3, 40, 64, 99], dtype=torch.int32)
    out, lse, ss = S.decode(dev(d.q), dev(d.k_cache), dev(d.v_cache), dev(d.cache_seqlens),
                            d.n_sink, d.window, dev(d.sink), scale=d.scale, num_splits=splits)
    torch.cuda.synchronize()
    assert out.dtype == F16
    ro, rl, rs = oracle.decode(d.q, d.k_cache, d.v_cache, d.cache_seqlens, d.n_sink, d.window,
                               d.sink, d.scale)
    tol = TOL[F16]
    assert max_abs(np64(out), ro) <= tol["o"]
    check_lse(np64(lse), rl, tol["lse"])
    assert max_abs(np64(ss), rs) <= tol["ss"]


def test_fp16_vanilla_gate():
    cu = [0, 300, 555]
    inp = W.make_attn("gate_f16", T_tot=555, Hq=8, Hkv=2, D=128, dtype=F16, mask=_spec(cu),
                      seed=47, sink_std=None)
    ref = oracle.gate_vanilla(inp.q, inp.k, inp.scale, **inp.mask.oracle_kwargs())
    _, rl, _ = oracle.fwd(inp.q, inp.k, inp.v, None, inp.scale, **inp.mask.oracle_kwargs())
    m = S.Mask.from_spec(inp.mask)
    got = S.gate_vanilla(dev(inp.q), dev(inp.k), torch.from_numpy(rl).float().cuda(), m,
                         scale=inp.scale)
    torch.cuda.synchronize()
    assert np.abs(np64(got) - ref).max() <= 2e-5
