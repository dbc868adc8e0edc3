"""Failure detection on the GPU without a fault: a barrier wait that can never
complete must end by itself with SINKATTN_ERR_TIMEOUT, and the context must
stay usable afterwards."""
import numpy as np
import pytest
import torch

import oracle
from learnable_sink_b200 import sinkattn as S
from learnable_sink_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.clear_status()
    S.selftest_timeout()
    assert S.get_status() == 5  # SINKATTN_ERR_TIMEOUT
    S.clear_status()
    assert S.get_status() == 0
    # the context is still usable: a forward call afterwards is correct
    inp = W.make_attn("after_timeout", T_tot=200, Hq=4, Hkv=2, D=128, dtype=torch.bfloat16,
                      mask=W.MaskSpec(causal=True, cu_seqlens=torch.tensor([0, 200], dtype=torch.int32)),
                      seed=77)
    m = S.Mask.from_spec(inp.mask)
    plan = S.Plan(200, 4, 2, m)
    out, lse, _ = S.fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.sink.cuda(), m, plan,
                        scale=inp.scale)
    torch.cuda.synchronize()
    ro, rl, _ = oracle.fwd(inp.q, inp.k, inp.v, inp.sink, inp.scale, **inp.mask.oracle_kwargs())
    assert np.abs(out.float().cpu().numpy() - ro).max() <= 2e-2
    assert S.get_status() == 0


def test_invalid_arguments_are_rejected_on_the_host():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    inp = W.tiny()
    m = S.Mask.from_spec(inp.mask)
    plan = S.Plan(128, 4, 2, m)
    q = inp.q.cuda()
    k3 = torch.empty(128, 3, 64, device="cuda")  # Hq % Hkv != 0
    with pytest.raises(S.SinkAttnError) as e:
        S.fwd(q, k3, k3, None, m, plan)
    assert e.value.code == 1
    bad = S.Mask(cu_seqlens=m.cu_seqlens, max_seqlen=128, causal=False, window=16)
    with pytest.raises(S.SinkAttnError):
        S.Plan(128, 4, 2, bad)  # a window needs the causal mask
    assert S.get_status() == 0
