"""GPU parity of the gate statistics and the gate-gradient backward against
the float64 oracle (page "Attention Sink and the native MoE in attention
layers", lvdousha26.github.io, sections 4-5: head importance is the mean gate
sink_s over tokens; the sink-aware balance loss trains through the gate, so
the backward takes an upstream gradient of sink_s)."""
import numpy as np
import pytest
import torch

import oracle
from learnable_sink_b200 import sinkattn as S
from learnable_sink_b200 import workloads as W

from gpu_util import TOL, check_status, dev, np64, rel_err, run_fwd

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.clear_status()
    yield
    check_status()


def spec(cu, n_sink=0, window=0):
    return W.MaskSpec(causal=True, n_sink=n_sink, window=window,
                      cu_seqlens=torch.tensor(cu, dtype=torch.int32))


# ------------------------------------------------------------ head importance

@pytest.mark.parametrize("T,Hq", [(1, 1), (31, 8), (33, 40), (1000, 3), (5000, 32),
                                  (32769, 64), (100003, 256)])
def test_importance_matches_oracle(T, Hq):
    ss, _ = W.gate_inputs(T, Hq, seed=T + Hq)
    got = S.gate_importance(ss.cuda())
    again = S.gate_importance(ss.cuda())
    torch.cuda.synchronize()
    ref = oracle.gate_importance(ss)
    # float64 partial sums of the same float32 values, rounded once to float32
    np.testing.assert_allclose(np64(got), ref, rtol=2e-7, atol=0)
    assert torch.equal(got, again), "importance is not bitwise reproducible"


def test_importance_rejects_bad_sizes():
    assert S.lib().sinkattn_gate_importance(0, 8, None, None, None, 0, None) == 1
    ss = torch.zeros(4, 257, device="cuda")
    imp = torch.zeros(257, device="cuda")
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    assert S.lib().sinkattn_gate_importance(4, 257, ss.data_ptr(), imp.data_ptr(), ws.data_ptr(),
                                            ws.numel(), None) == 2
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    ss = torch.zeros(100, 8, device="cuda")
    assert S.lib().sinkattn_gate_importance(100, 8, ss.data_ptr(), imp.data_ptr(),
                                            small.data_ptr(), small.numel(),
                                            None) == 4


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_importance_of_forward_gate(dtype):
    """Forward -> sink_s -> Imp on the GPU against the oracle's forward and mean."""
    mask = spec([0, 300, 555], n_sink=4, window=100)
    inp = W.make_attn("imp", T_tot=555, Hq=8, Hkv=2, D=128, dtype=dtype, mask=mask, seed=41)
    _, _, ss, _, _ = run_fwd(inp)
    got = np64(S.gate_importance(ss))
    _, _, rs = oracle.fwd(inp.q, inp.k, inp.v, inp.sink, inp.scale, **mask.oracle_kwargs())
    np.testing.assert_allclose(got, oracle.gate_importance(rs), atol=TOL[dtype]["ss"], rtol=0)


# ------------------------------------------------------ gate-gradient backward

def _bwd_with_gate_grad(inp, dss, out, lse, m, plan):
    r = S.bwd(dev(inp.q), dev(inp.k), dev(inp.v), out, dev(inp.dout), lse, dev(inp.sink), m,
              plan, scale=inp.scale, d_sink_s=dss.cuda().contiguous())
    torch.cuda.synchronize()
    return r


def _check(inp, dss, grads):
    tol = TOL[inp.q.dtype]
    r = oracle.bwd(inp.q, inp.k, inp.v, inp.sink, inp.dout, inp.scale, dss=dss,
                   **inp.mask.oracle_kwargs())
    for name, got, ref in (("dq", grads[0], r[0]), ("dk", grads[1], r[1]), ("dv", grads[2], r[2])):
        e = rel_err(np64(got), ref)
        assert e <= tol["grad"], f"{name} rel {e:.3e}"
    if inp.sink is not None:
        e = rel_err(np64(grads[3]), r[3])
        assert e <= tol["grad"], f"dsink rel {e:.3e}"
    return r


GATE_CASES = {
    "fp32_causal_ragged": dict(cu=[0, 130, 300], Hq=4, Hkv=2, D=64, dtype=torch.float32),
    "fp32_extreme_sinks": dict(cu=[0, 300], Hq=4, Hkv=2, D=64, dtype=torch.float32,
                               sink_values=[-30.0, -2.0, 2.0, 30.0]),
    "bf16_causal_D128_G4": dict(cu=[0, 300, 555], Hq=8, Hkv=2, D=128, dtype=torch.bfloat16),
    "bf16_band_D64": dict(cu=[0, 260, 700], Hq=8, Hkv=4, D=64, dtype=torch.bfloat16,
                          n_sink=4, window=37),
    "bf16_no_sink": dict(cu=[0, 333], Hq=4, Hkv=2, D=128, dtype=torch.bfloat16, sink_std=None),
}


@pytest.mark.parametrize("name", list(GATE_CASES))
def test_gate_gradient_backward(name):
    kw = dict(GATE_CASES[name])
    cu = kw.pop("cu")
    mask = spec(cu, kw.pop("n_sink", 0), kw.pop("window", 0))
    T = cu[-1]
    inp = W.make_attn(name, T_tot=T, mask=mask, seed=43, **kw)
    _, dss = W.gate_inputs(T, kw["Hq"], seed=44)
    dss = dss * 4.0
    out, lse, _, m, plan = run_fwd(inp)
    _check(inp, dss, _bwd_with_gate_grad(inp, dss, out, lse, m, plan))


@pytest.mark.parametrize("n_shared", [0, 2])
def test_balance_loss_gradient_through_backward(n_shared):
    """The upstream gradient of the sink-aware balance loss, d loss / d Imp_h
    spread over the tokens (d Imp_h / d sink_s[t, h] = 1 / T), taken from the
    oracle's forward and loss, through the GPU backward with dout = 0: dsink
    and dQ/dK come from the gate alone, dV is zero."""
    mask = spec([0, 384, 640])
    inp = W.make_attn("aux", T_tot=640, Hq=8, Hkv=2, D=128, dtype=torch.bfloat16, mask=mask,
                      seed=45)
    inp.dout = torch.zeros_like(inp.dout)
    _, _, rs = oracle.fwd(inp.q, inp.k, inp.v, inp.sink, inp.scale, **mask.oracle_kwargs())
    _, d_imp = oracle.gate_aux_loss(oracle.gate_importance(rs), lam=1.0, n_shared=n_shared)
    dss = torch.from_numpy(np.broadcast_to(d_imp / 640.0, (640, 8)).copy()).float()
    out, lse, _, m, plan = run_fwd(inp)
    grads = _bwd_with_gate_grad(inp, dss, out, lse, m, plan)
    _check(inp, dss, grads)
    assert float(grads[2].abs().max()) == 0.0


# ------------------------------------------------------ gate of a sink-free model

VANILLA_CASES = {
    "bf16_causal_ragged_D128": dict(cu=[0, 300, 555], Hq=8, Hkv=2, D=128, dtype=torch.bfloat16),
    "bf16_band_no_sink_tokens": dict(cu=[0, 200, 333], Hq=4, Hkv=2, D=64, dtype=torch.bfloat16,
                                     window=37),
    "bf16_band_with_sink_tokens": dict(cu=[0, 260], Hq=8, Hkv=1, D=128, dtype=torch.bfloat16,
                                       n_sink=4, window=50),
    "fp32_causal_D64": dict(cu=[0, 1, 130, 300], Hq=4, Hkv=4, D=64, dtype=torch.float32),
    "bf16_block_sparse": dict(cu=None, Hq=8, Hkv=2, D=64, dtype=torch.bfloat16),
}


def _vanilla_inputs(name):
    kw = dict(VANILLA_CASES[name])
    cu = kw.pop("cu")
    if cu is None:
        cu_t = torch.tensor([0, 200, 450, 700], dtype=torch.int32)
        bi = W.random_block_indices(cu_t, kw["Hkv"], 64, 64, 2, 51)
        bi[:, 1, :] = torch.where(bi[:, 1, :] == 0, -1, bi[:, 1, :])  # a block that skips k_0
        mask = W.MaskSpec(causal=True, cu_seqlens=cu_t, block_indices=bi, block_q=64, block_k=64)
        T = 700
    else:
        mask = spec(cu, kw.pop("n_sink", 0), kw.pop("window", 0))
        T = cu[-1]
    return W.make_attn(name, T_tot=T, mask=mask, seed=52, sink_std=None, **kw)


@pytest.mark.parametrize("name", list(VANILLA_CASES))
def test_vanilla_gate(name):
    inp = _vanilla_inputs(name)
    ref = oracle.gate_vanilla(inp.q, inp.k, inp.scale, **inp.mask.oracle_kwargs())
    m = S.Mask.from_spec(inp.mask)
    # the gate kernel alone, on the oracle's sink-free LSE
    _, rl, _ = oracle.fwd(inp.q, inp.k, inp.v, None, inp.scale, **inp.mask.oracle_kwargs())
    lse = torch.from_numpy(rl).float().cuda()
    got = S.gate_vanilla(dev(inp.q), dev(inp.k), lse, m, scale=inp.scale)
    torch.cuda.synchronize()
    assert np.abs(np64(got) - ref).max() <= 2e-5
    # through the library's own sink-free forward
    _, lse_f, _, m, _ = run_fwd(inp)
    got = S.gate_vanilla(dev(inp.q), dev(inp.k), lse_f, m, scale=inp.scale)
    torch.cuda.synchronize()
    err = np.abs(np64(got) - ref).max()
    assert err <= TOL[inp.q.dtype]["ss"], f"gate max abs {err:.3e}"
