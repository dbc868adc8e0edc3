"""The no-allocation decode entry point (sinkattn_decode_noalloc).

It serves callers that cannot provide scratch memory -- a serving loop that
reserves all device memory up front and may not allocate mid-request, or a
plain C program that owns only its inputs and outputs -- from a fixed scratch
array inside the library.  Each case runs two calls in a row (the second sees
the first's leftovers in the shared array) and compares both with the float64
oracle and with the workspace entry point.  This file is collected last so
that a run stopping at the first failure has already run every other test; it
also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from learnable_sink_b200 import sinkattn as S
from learnable_sink_b200 import workloads as W

from gpu_util import TOL, check_lse, max_abs, np64

pytestmark = pytest.mark.gpu

_vp, _i = ctypes.c_void_p, ctypes.c_int


def _fn():
    f = S.lib().sinkattn_decode_noalloc
    f.argtypes = [_i, _i, _i, _i, _i, ctypes.c_float, _vp, _vp, _vp, _vp, _i, _i, _vp, _vp, _vp,
                  _vp, _i, _vp]
    f.restype = _i
    return f


def _p(t):
    return None if t is None else _vp(t.data_ptr())


def _outputs(d):
    B, Hq, D = d.q.shape
    out = torch.empty(B, Hq, D, dtype=d.q.dtype, device="cuda")
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    return out, lse, torch.empty_like(lse)


def _call_noalloc(d, t, outs, num_splits=0):
    B, Hq, D = d.q.shape
    Hkv = d.k_cache.shape[2]
    out, lse, ss = outs
    dt = S.BF16 if d.q.dtype == torch.bfloat16 else S.FP32
    return _fn()(dt, B, Hq, Hkv, D, d.scale, _p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["cs"]),
                 d.n_sink, d.window, _p(t["sink"]), _p(out), _p(lse), _p(ss), num_splits,
                 _vp(torch.cuda.current_stream().cuda_stream))


def _dev(d):
    return {"q": d.q.cuda(), "k": d.k_cache.cuda(), "v": d.v_cache.cuda(),
            "cs": d.cache_seqlens.cuda(), "sink": None if d.sink is None else d.sink.cuda()}


CASES = {
    # the StreamingLLM config: 32 sequences, 4 + 1020 slots, Hq 32, Hkv 8, D 128
    "streamingllm_bf16": lambda: W.decode(),
    # ragged, partly filled caches, D 64
    "ragged_bf16_d64": lambda: W.decode(B=5, n_sink=4, window=200, Hq=16, Hkv=4, D=64,
                                        seqlen_range=(1, 400), seed_offset=7),
    # the fp32 split kernel through the same shared array
    "ragged_fp32": lambda: W.decode(B=4, n_sink=2, window=90, Hq=8, Hkv=2, D=128,
                                    dtype=torch.float32, seqlen_range=(0, 200), seed_offset=8),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("num_splits", [0, 3, 10 ** 6])  # automatic, explicit, clamped
def test_noalloc_decode_matches_oracle_and_workspace_decode_twice(case, num_splits):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.clear_status()
    d = CASES[case]()
    tol = TOL[d.q.dtype]
    t = _dev(d)
    ro, rl, rs = oracle.decode(d.q, d.k_cache, d.v_cache, d.cache_seqlens, d.n_sink, d.window,
                               d.sink, d.scale)
    ref = S.decode(t["q"], t["k"], t["v"], t["cs"], d.n_sink, d.window, t["sink"],
                   scale=d.scale)
    outs = [_outputs(d), _outputs(d)]
    B, Hq, D = d.q.shape
    if num_splits > 0:
        # an explicit count is first lowered like the workspace decode's
        # (to the 16-row pieces of one pair, at most 128); if the partials
        # then exceed the 4 MiB array the call is refused before any launch
        n = min(num_splits, -(-(d.n_sink + d.window) // 16), 128)
        if -(-(4 * B * Hq * n * (D + 2)) // 256) * 256 > 4 << 20:
            assert _call_noalloc(d, t, outs[0], num_splits) == 4  # SINKATTN_ERR_WORKSPACE
            return
    # first call: looks up the array's address (and loads the kernels)
    assert _call_noalloc(d, t, outs[0], num_splits) == 0
    torch.cuda.synchronize()
    free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for k in range(2):  # two calls in a row; the second sees the first's leftovers
        rc = _call_noalloc(d, t, outs[k], num_splits)
        torch.cuda.synchronize()
        assert rc == 0, S.error_string(rc)
    # nothing was allocated by those calls
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    for out, lse, ss in outs:
        assert max_abs(np64(out), ro) <= tol["o"]
        check_lse(np64(lse), rl, tol["lse"])
        assert max_abs(np64(ss), rs) <= tol["ss"]
        assert max_abs(np64(out), np64(ref[0])) <= tol["o"]
        assert max_abs(np64(ss), np64(ref[2])) <= tol["ss"]
    assert S.get_status() == 0


def test_noalloc_decode_rejects_oversize_problem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = W.decode(B=2, n_sink=4, window=60, Hq=8, Hkv=2, D=128, seqlen_range=(1, 64))
    t = _dev(d)
    # 4096 sequences x 64 heads x 8 slots x 130 floats is far beyond 4 MiB:
    # rejected on the host before anything is launched
    rc = _fn()(S.BF16, 4096, 64, 8, 128, d.scale, _p(t["q"]), _p(t["k"]), _p(t["v"]),
               _p(t["cs"]), 4, 1020, _p(t["sink"]), _p(t["q"]), _p(t["cs"]), None, 8,
               _vp(torch.cuda.current_stream().cuda_stream))
    assert rc == 4  # SINKATTN_ERR_WORKSPACE
