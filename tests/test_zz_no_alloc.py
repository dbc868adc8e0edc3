"""The no-allocation decode entry point (sinkattn_decode_noalloc).

It serves callers that cannot provide scratch memory -- a serving loop that
reserves all device memory up front and may not allocate mid-request, or a
plain C program that owns only its inputs and outputs -- from a fixed scratch
array inside the library.  This file is collected last so that a run stopping
at the first failure has already run every other test; it also passes alone in
a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from learnable_sink_b200 import sinkattn as S
from learnable_sink_b200 import workloads as W

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


def _call_noalloc(d, t, num_splits=0):
    B, Hq, D = d.q.shape
    Hkv = d.k_cache.shape[2]
    out = torch.empty_like(t["q"])
    lse = torch.empty(B, Hq, dtype=torch.float32, device="cuda")
    ss = torch.empty_like(lse)
    rc = _fn()(S.BF16, B, Hq, Hkv, D, d.scale, _p(t["q"]), _p(t["k"]), _p(t["v"]), _p(t["cs"]),
               d.n_sink, d.window, _p(t["sink"]), _p(out), _p(lse), _p(ss), num_splits,
               _vp(torch.cuda.current_stream().cuda_stream))
    return rc, out, lse, ss


def _dev(d):
    return {"q": d.q.cuda(), "k": d.k_cache.cuda(), "v": d.v_cache.cuda(),
            "cs": d.cache_seqlens.cuda(), "sink": None if d.sink is None else d.sink.cuda()}


def test_noalloc_decode_matches_workspace_decode_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.clear_status()
    cases = [W.decode(),  # 32 sequences, 4 + 1020 slots, Hq 32, Hkv 8, D 128
             W.decode(B=5, n_sink=4, window=200, Hq=16, Hkv=4, D=64, seqlen_range=(1, 400),
                      seed_offset=7)]
    for d in cases:  # two calls in a row; the second sees the first's leftovers
        t = _dev(d)
        ref = S.decode(t["q"], t["k"], t["v"], t["cs"], d.n_sink, d.window, t["sink"],
                       scale=d.scale)
        rc, out, lse, ss = _call_noalloc(d, t)
        torch.cuda.synchronize()
        assert rc == 0, S.error_string(rc)
        o1, o2 = ref[0].float().cpu().numpy(), out.float().cpu().numpy()
        assert np.abs(o1 - o2).max() <= 2e-2
        assert np.abs(ref[1].cpu().numpy() - lse.cpu().numpy()).max() <= 1e-3
        assert np.abs(ref[2].cpu().numpy() - ss.cpu().numpy()).max() <= 1e-3
    assert S.get_status() == 0


def test_noalloc_decode_rejects_oversize_problem():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    d = W.decode(B=2, n_sink=4, window=60, Hq=8, Hkv=2, D=128, seqlen_range=(1, 64))
    t = _dev(d)
    # 4096 sequences x 64 heads x 8 splits x 130 floats is far beyond 4 MiB:
    # rejected on the host before anything is launched
    rc = _fn()(S.BF16, 4096, 64, 8, 128, d.scale, _p(t["q"]), _p(t["k"]), _p(t["v"]),
               _p(t["cs"]), 4, 1020, _p(t["sink"]), _p(t["q"]), _p(t["cs"]), None, 8,
               _vp(torch.cuda.current_stream().cuda_stream))
    assert rc == 4  # SINKATTN_ERR_WORKSPACE
