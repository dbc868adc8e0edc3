"""Ring-cache maintenance (page "Attention Sink / StreamingLLM", core idea:
fixed sink slots plus a circular window whose oldest entry is overwritten).

The expected cache is built here from the slot rule, token by token in
logical order (a later token overwrites an earlier one in the same slot), and
the GPU caches must match it bit-exactly (these are copies).  Decode over an
appended cache is then checked against the oracle's forward of the last token
of the full logical sequence under the matching StreamingLLM band mask
(n_sink sink keys + a causal window), which ties the ring layout to the
attention it stands for.
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


def slot_of(p, n_sink, window):
    if p < n_sink:
        return p
    return None if window == 0 else n_sink + (p - n_sink) % window


def ring_of(seq, n_sink, window, base):
    """Expected cache [S, Hkv, D] after appending the tokens of seq in order,
    starting from `base` (slots never written keep their base content)."""
    out = base.clone()
    for p in range(seq.shape[0]):
        s = slot_of(p, n_sink, window)
        if s is not None:
            out[s] = seq[p]
    return out


def _gen(shape, seed, dtype):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(dtype)


@pytest.mark.parametrize("dtype,D,n_sink,window", [(torch.bfloat16, 128, 4, 64),
                                                    (torch.float32, 64, 2, 30),
                                                    (torch.bfloat16, 64, 3, 0)])
def test_fill_then_append_matches_slot_rule(dtype, D, n_sink, window):
    Hkv = 2
    lens = [0, 1, 5, 37, 300]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    k = _gen((T, Hkv, D), 1, dtype)
    v = _gen((T, Hkv, D), 2, dtype)
    S_ = n_sink + window
    n_seq = len(lens)
    base_k = _gen((n_seq, S_, Hkv, D), 3, dtype)
    base_v = _gen((n_seq, S_, Hkv, D), 4, dtype)
    kc, vc = dev(base_k), dev(base_v)
    lens_out = torch.full((n_seq,), -7, dtype=torch.int32, device="cuda")
    S.cache_fill(dev(k), dev(v), dev(torch.from_numpy(cu)), kc, vc, n_sink, window, lens_out)
    torch.cuda.synchronize()
    assert lens_out.cpu().tolist() == lens
    for s in range(n_seq):
        a, b = int(cu[s]), int(cu[s + 1])
        assert torch.equal(kc[s].cpu(), ring_of(k[a:b], n_sink, window, base_k[s]))
        assert torch.equal(vc[s].cpu(), ring_of(v[a:b], n_sink, window, base_v[s]))
    # append 70 more tokens to every sequence, one step at a time
    n_new = 70
    k_new = _gen((n_new, n_seq, Hkv, D), 5, dtype)
    v_new = _gen((n_new, n_seq, Hkv, D), 6, dtype)
    seqlens = torch.tensor(lens, dtype=torch.int32)
    for t in range(n_new):
        seqlens += 1
        S.cache_append(dev(k_new[t]), dev(v_new[t]), dev(seqlens), kc, vc, n_sink, window)
    torch.cuda.synchronize()
    for s in range(n_seq):
        a, b = int(cu[s]), int(cu[s + 1])
        full_k = torch.cat([k[a:b], k_new[:, s]])
        full_v = torch.cat([v[a:b], v_new[:, s]])
        assert torch.equal(kc[s].cpu(), ring_of(full_k, n_sink, window, base_k[s]))
        assert torch.equal(vc[s].cpu(), ring_of(full_v, n_sink, window, base_v[s]))


def test_append_skips_empty_and_decode_over_appended_cache():
    n_sink, window, Hq, Hkv, D = 4, 96, 8, 2, 128
    lens = [10, 150, 500]                       # the longest wraps the window many times
    B = len(lens)
    S_ = n_sink + window
    seqs = [_gen((L, Hkv, D), 10 + i, torch.bfloat16) for i, L in enumerate(lens)]
    vals = [_gen((L, Hkv, D), 20 + i, torch.bfloat16) for i, L in enumerate(lens)]
    kc = torch.zeros(B, S_, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    seqlens = torch.zeros(B, dtype=torch.int32)
    for t in range(max(lens)):
        kn = torch.zeros(B, Hkv, D, dtype=torch.bfloat16)
        vn = torch.zeros_like(kn)
        active = torch.tensor([t < L for L in lens])
        for b in range(B):
            if active[b]:
                kn[b], vn[b] = seqs[b][t], vals[b][t]
        seqlens = seqlens + active.to(torch.int32)
        # a sequence that has no new token passes its old count: the append
        # rewrites its latest token with itself only if the count is > 0, so
        # finished sequences are given 0 here and must stay untouched
        sl = torch.where(active, seqlens, torch.zeros_like(seqlens))
        S.cache_append(dev(kn), dev(vn), dev(sl), kc, vc, n_sink, window)
    torch.cuda.synchronize()
    q = _gen((B, Hq, D), 30, torch.bfloat16)
    sink = _gen((Hq,), 31, torch.float32)
    scale = 1.0 / np.sqrt(D)
    out, lse, ss = S.decode(dev(q), kc, vc, dev(seqlens), n_sink, window, dev(sink), scale=scale)
    torch.cuda.synchronize()
    tol = TOL[torch.bfloat16]
    for b, L in enumerate(lens):
        # the last token's query over the whole logical sequence, band mask
        qq = torch.zeros(L, Hq, D, dtype=torch.bfloat16)
        qq[L - 1] = q[b]
        rows = np.array([[L - 1, h] for h in range(Hq)], dtype=np.int32)
        ro, rl, rs = oracle.fwd_rows(qq, seqs[b], vals[b], sink, scale, rows, causal=True,
                                     n_sink=n_sink, window=window,
                                     cu_seqlens=torch.tensor([0, L], dtype=torch.int32))
        assert np.abs(np64(out[b]) - ro).max() <= tol["o"]
        assert np.abs(np64(lse[b]) - rl).max() <= tol["lse"]
        assert np.abs(np64(ss[b]) - rs).max() <= tol["ss"]
