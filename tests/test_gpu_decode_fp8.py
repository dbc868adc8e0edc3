"""GPU parity of the mixed-precision ring decode (sinkattn_decode_fp8): bf16
sink slots, FP8 E4M3 window slots with per-KV-head scales (page "Attention
Sink / StreamingLLM", on KV-cache quantisation: keep the first tokens in high
precision).  Compared element by element with the float64 oracle
(oracle.decode_fp8_window) on the same codes and scales, at the bf16
tolerances."""
import numpy as np
import pytest
import torch

import oracle
from learnable_sink_b200 import sinkattn as S
from learnable_sink_b200 import workloads as W

from gpu_util import TOL, check_lse, check_status, max_abs, np64

pytestmark = pytest.mark.gpu


def _run(d, cache, num_splits=0):
    ks, vs, kw, vw, ksc, vsc = (t.cuda().contiguous() for t in cache)
    out, lse, ss = S.decode_fp8(d.q.cuda(), ks, vs, kw, vw, ksc, vsc, d.cache_seqlens.cuda(),
                                d.n_sink, d.window, None if d.sink is None else d.sink.cuda(),
                                scale=d.scale, num_splits=num_splits)
    torch.cuda.synchronize()
    return out, lse, ss


def _compare(d, cache, got, tol=TOL[torch.bfloat16]):
    ks, vs, kw, vw, ksc, vsc = cache
    ro, rl, rs = oracle.decode_fp8_window(d.q, ks, vs, kw, vw, ksc, vsc, d.cache_seqlens,
                                          d.n_sink, d.window, d.sink, d.scale)
    out, lse, ss = got
    assert max_abs(np64(out), ro) <= tol["o"]
    check_lse(np64(lse), rl, tol["lse"])
    assert max_abs(np64(ss), rs) <= tol["ss"]


def test_fp8_decode_streamingllm_config():
    """32 sequences, 4 bf16 sink slots + 1020 FP8 window slots, Hq 32, Hkv 8,
    D 128, every slot filled, ring heads at random positions."""
    S.clear_status()
    d = W.decode()
    cache = W.fp8_window_cache(d, seed=W.SEED_BASE + 501)
    _compare(d, cache, _run(d, cache))
    check_status()


@pytest.mark.parametrize("splits", [0, 1, 2, 3, 40])
@pytest.mark.parametrize("D", [64, 128])
def test_fp8_decode_partial_fill_and_splits(D, splits):
    """Ragged, partly filled caches (some shorter than the sink segment, one
    empty) and a window that is not a multiple of the 32-row pieces."""
    S.clear_status()
    d = W.decode(B=7, n_sink=4, window=200, Hq=8, Hkv=2, D=D, seqlen_range=(0, 260),
                 seed_offset=31)
    d.cache_seqlens[0] = 0
    d.cache_seqlens[1] = 3
    cache = W.fp8_window_cache(d, seed=W.SEED_BASE + 502)
    _compare(d, cache, _run(d, cache, splits))
    check_status()


@pytest.mark.parametrize("G", [1, 2, 8])
@pytest.mark.parametrize("n_sink", [0, 20])
def test_fp8_decode_heads_and_sink_segments(G, n_sink):
    """No sink slots at all, or a sink segment spanning two 16-row pieces;
    1, 2 and 8 query heads per KV head."""
    S.clear_status()
    d = W.decode(B=5, n_sink=n_sink, window=300, Hq=2 * G, Hkv=2, D=128,
                 seqlen_range=(1, 700), seed_offset=32 + G + n_sink)
    cache = W.fp8_window_cache(d, seed=W.SEED_BASE + 503)
    if n_sink == 0:
        cache = (None, None) + tuple(cache[2:])
        ks, vs, kw, vw, ksc, vsc = cache
        out, lse, ss = S.decode_fp8(d.q.cuda(), None, None, kw.cuda(), vw.cuda(), ksc.cuda(),
                                    vsc.cuda(), d.cache_seqlens.cuda(), 0, d.window,
                                    d.sink.cuda(), scale=d.scale)
        torch.cuda.synchronize()
        z = torch.zeros(d.q.shape[0], 0, d.k_cache.shape[2], d.q.shape[2], dtype=torch.bfloat16)
        _compare(d, (z, z, kw, vw, ksc, vsc), (out, lse, ss))
    else:
        _compare(d, cache, _run(d, cache))
    check_status()


def test_fp8_decode_ignores_nan_in_unfilled_slots():
    """Unfilled sink slots hold NaN and unfilled window slots hold the NaN
    code: neither reaches the outputs."""
    S.clear_status()
    d = W.decode(B=6, n_sink=4, window=100, Hq=8, Hkv=2, D=128, seqlen_range=(0, 60),
                 seed_offset=41)
    ks, vs, kw, vw, ksc, vsc = W.fp8_window_cache(d, seed=W.SEED_BASE + 504)
    cs = d.cache_seqlens.tolist()
    for b, n in enumerate(cs):
        if n < 4:
            ks[b, n:] = float("nan")
            vs[b, n:] = float("nan")
        w = max(n - 4, 0)
        kw[b, w:] = 0x7F
        vw[b, w:] = 0xFF
    cache = (ks, vs, kw, vw, ksc, vsc)
    got = _run(d, cache)
    for t in got:
        assert not torch.isnan(t.float()).any()
    # the oracle dequantises NaN codes to NaN; compare on the filled slots only
    clean = (ks.nan_to_num(0.0), vs.nan_to_num(0.0), torch.where(kw == 0x7F, 0, kw).to(torch.uint8),
             torch.where(vw == 0xFF, 0, vw).to(torch.uint8), ksc, vsc)
    _compare(d, clean, got)
    check_status()


def test_fp8_decode_matches_bf16_decode_of_dequantised_cache():
    """The FP8 decode equals sinkattn_decode run on the same cache
    dequantised to bf16 where dequantisation is exact in bf16 (E4M3 codes
    times power-of-two scales)."""
    S.clear_status()
    d = W.decode(B=4, n_sink=4, window=124, Hq=16, Hkv=4, D=128, seqlen_range=(100, 400),
                 seed_offset=42)
    ks, vs, kw, vw, _, _ = W.fp8_window_cache(d, seed=W.SEED_BASE + 505)
    ksc = torch.tensor([2.0 ** -4, 2.0 ** -5, 2.0 ** -3, 2.0 ** -6], dtype=torch.float32)
    vsc = torch.tensor([2.0 ** -5, 2.0 ** -4, 2.0 ** -6, 2.0 ** -3], dtype=torch.float32)
    deq_k = torch.from_numpy(oracle.fp8_e4m3_value(kw.numpy())) * ksc.double()[None, None, :, None]
    deq_v = torch.from_numpy(oracle.fp8_e4m3_value(vw.numpy())) * vsc.double()[None, None, :, None]
    kc = torch.cat([ks, deq_k.to(torch.bfloat16)], dim=1)
    vc = torch.cat([vs, deq_v.to(torch.bfloat16)], dim=1)
    assert torch.equal(kc[:, 4:].double(), deq_k)  # exact in bf16
    got = _run(d, (ks, vs, kw, vw, ksc, vsc))
    ref = S.decode(d.q.cuda(), kc.cuda(), vc.cuda(), d.cache_seqlens.cuda(), d.n_sink, d.window,
                   d.sink.cuda(), scale=d.scale)
    torch.cuda.synchronize()
    assert max_abs(np64(got[0]), np64(ref[0])) <= 2e-2
    assert max_abs(np64(got[1]), np64(ref[1])) <= 1e-3
    assert max_abs(np64(got[2]), np64(ref[2])) <= 1e-3
    check_status()


@pytest.mark.parametrize("D", [64, 128])
def test_fp8_cache_append_bit_exact_then_decode(D):
    """Appends into the mixed-precision cache are bit-exact against the
    oracle's slot rule and E4M3 encoder (positions in the sink segment, in
    the window, past a wrap, and an empty sequence); a decode over the
    appended cache then matches the oracle."""
    S.clear_status()
    d = W.decode(B=6, n_sink=4, window=40, Hq=8, Hkv=2, D=D, seqlen_range=(0, 200),
                 seed_offset=51)
    ks, vs, kw, vw, ksc, vsc = W.fp8_window_cache(d, seed=W.SEED_BASE + 506)
    gen = torch.Generator().manual_seed(W.SEED_BASE + 507)
    B, Hkv = d.q.shape[0], d.k_cache.shape[2]
    cs = torch.tensor([0, 1, 4, 5, 44, 173], dtype=torch.int32)  # positions -1, 0, 3, 4, 43, 172
    kn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
    vn = torch.randn(B, Hkv, D, generator=gen).to(torch.bfloat16)
    kn[5, 0, :4] = torch.tensor([1e4, -1e4, 0.0, -0.0], dtype=torch.bfloat16)  # saturation, signed 0
    ref = oracle.cache_append_fp8(kn, vn, cs, ks, vs, kw, vw, ksc, vsc, d.n_sink, d.window)
    dev = [t.cuda().contiguous() for t in (ks, vs, kw, vw, ksc, vsc)]
    S.cache_append_fp8(kn.cuda(), vn.cuda(), cs.cuda(), dev[0], dev[1], dev[2], dev[3], dev[4],
                       dev[5], d.n_sink, d.window)
    torch.cuda.synchronize()
    assert np.array_equal(dev[0].float().cpu().double().numpy(), ref[0])
    assert np.array_equal(dev[1].float().cpu().double().numpy(), ref[1])
    assert np.array_equal(dev[2].cpu().numpy(), ref[2])
    assert np.array_equal(dev[3].cpu().numpy(), ref[3])
    # decode over the appended cache, every sequence at its new length
    out, lse, ss = S.decode_fp8(d.q.cuda(), dev[0], dev[1], dev[2], dev[3], dev[4], dev[5],
                                cs.cuda(), d.n_sink, d.window, d.sink.cuda(), scale=d.scale)
    torch.cuda.synchronize()
    ro, rl, rs = oracle.decode_fp8_window(d.q, ref[0], ref[1], ref[2], ref[3], ksc, vsc, cs,
                                          d.n_sink, d.window, d.sink, d.scale)
    tol = TOL[torch.bfloat16]
    assert max_abs(np64(out), ro) <= tol["o"]
    check_lse(np64(lse), rl, tol["lse"])
    assert max_abs(np64(ss), rs) <= tol["ss"]
    check_status()
