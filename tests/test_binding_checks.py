"""The Python binding refuses, before any launch, argument metadata the C ABI
cannot see through raw pointers (element types and extents), and accepts the
argument patterns the GPU tests and the benchmark use.  CPU tensors: a call
whose metadata is valid stops at the device check instead."""
import pytest
import torch

from learnable_sink_b200 import sinkattn as S

T, Hq, Hkv, D = 64, 8, 2, 128
bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def _mask():
    return S.Mask(cu_seqlens=torch.tensor([0, 40, 64], dtype=i32), max_seqlen=40)


def _qkv(dtype=bf):
    return (torch.zeros(T, Hq, D, dtype=dtype), torch.zeros(T, Hkv, D, dtype=dtype),
            torch.zeros(T, Hkv, D, dtype=dtype))


def _passes_metadata(call):
    with pytest.raises(ValueError, match="contiguous CUDA tensors"):
        call()


def _refused(call, what):
    with pytest.raises(S.SinkAttnError, match=what) as e:
        call()
    assert e.value.code == 1


def test_valid_patterns_pass_the_metadata_checks():
    q, k, v = _qkv()
    sink, lse = torch.zeros(Hq, dtype=f32), torch.zeros(T, Hq, dtype=f32)
    m = _mask()
    _passes_metadata(lambda: S.fwd(q, k, v, sink, m, None, out=torch.empty_like(q), lse=lse,
                                   sink_s=torch.empty_like(lse), lse_orig=torch.empty_like(lse)))
    _passes_metadata(lambda: S.fwd(q, k, v, None, m, None))
    _passes_metadata(lambda: S.bwd(q, k, v, q, q, lse, sink, m, None, dq=torch.empty_like(q),
                                   dk=torch.empty_like(k), dv=torch.empty_like(v),
                                   dsink=torch.empty_like(sink), d_sink_s=lse))
    _passes_metadata(lambda: S.gate_importance(lse, imp=torch.empty(Hq)))
    _passes_metadata(lambda: S.gate_vanilla(q, k, lse, m, gate=torch.empty_like(lse)))
    B, n_sink, window = 5, 4, 60
    kc = torch.zeros(B, n_sink + window, Hkv, D, dtype=bf)
    cs = torch.zeros(B, dtype=i32)
    _passes_metadata(lambda: S.decode(torch.zeros(B, Hq, D, dtype=bf), kc, kc.clone(), cs,
                                      n_sink, window, sink, out=torch.zeros(B, Hq, D, dtype=bf),
                                      lse=torch.zeros(B, Hq), sink_s=torch.zeros(B, Hq)))
    kn = torch.zeros(B, Hkv, D, dtype=bf)
    _passes_metadata(lambda: S.cache_append(kn, kn.clone(), cs, kc, kc.clone(), n_sink, window))
    cu = torch.tensor([0, 10, 30, 30, 50, 64], dtype=i32)
    _passes_metadata(lambda: S.cache_fill(k, v, cu, kc, kc.clone(), n_sink, window, cs))


def test_attention_metadata_mismatches_are_refused():
    q, k, v = _qkv()
    m = _mask()
    sink, lse = torch.zeros(Hq, dtype=f32), torch.zeros(T, Hq, dtype=f32)
    _refused(lambda: S.fwd(q, k.float(), v, sink, m, None), "k is torch.float32")
    _refused(lambda: S.fwd(q, k, v[:, :1], sink, m, None), "k and v shapes differ")
    _refused(lambda: S.fwd(q, k[:32], v[:32], sink, m, None), "disagree on T or D")
    _refused(lambda: S.fwd(q, k, v, sink.half(), m, None), "learnable_sink")
    _refused(lambda: S.fwd(q, k, v, sink[:4], m, None), "learnable_sink")
    _refused(lambda: S.fwd(q, k, v, sink, m, None, out=q.float()), "out")
    _refused(lambda: S.fwd(q, k, v, sink, m, None, lse=lse[:, :4]), "lse")
    bad = S.Mask(cu_seqlens=torch.tensor([0, 64], dtype=torch.int64), max_seqlen=64)
    _refused(lambda: S.fwd(q, k, v, sink, bad, None), "cu_seqlens must be int32")
    _refused(lambda: S.bwd(q, k, v, q, q.float(), lse, sink, m, None), "dout")
    _refused(lambda: S.bwd(q, k, v, q, q, lse, sink, m, None, dk=torch.empty_like(q)), "dk")
    _refused(lambda: S.bwd(q, k, v, q, q, lse, sink, m, None, d_sink_s=lse.double()),
             "d_sink_s")
    _refused(lambda: S.bwd(q, k, v, q, q, lse, sink, m, None, dsink=torch.zeros(Hq + 1)),
             "dsink")
    _refused(lambda: S.gate_importance(lse.half()), "sink_s must be float32")
    _refused(lambda: S.gate_importance(lse, imp=torch.zeros(Hq + 1)), "imp")
    _refused(lambda: S.gate_vanilla(q, k, lse.T.contiguous(), m), "lse")


def test_ring_cache_metadata_mismatches_are_refused():
    B, n_sink, window = 5, 4, 60
    q = torch.zeros(B, Hq, D, dtype=bf)
    kc = torch.zeros(B, n_sink + window, Hkv, D, dtype=bf)
    cs = torch.zeros(B, dtype=i32)
    sink = torch.zeros(Hq)
    _refused(lambda: S.decode(q, kc, kc, cs, n_sink, window + 1, sink), "expected")
    _refused(lambda: S.decode(q, kc.float(), kc.float(), cs, n_sink, window, sink), "k_cache")
    _refused(lambda: S.decode(q, kc, kc, cs.long(), n_sink, window, sink), "cache_seqlens")
    _refused(lambda: S.decode(q, kc, kc[:, :, :1], cs, n_sink, window, sink), "shapes differ")
    kn = torch.zeros(B, Hkv, D, dtype=bf)
    _refused(lambda: S.cache_append(kn, kn.float(), cs, kc, kc, n_sink, window), "v_new")
    _refused(lambda: S.cache_append(kn[:, :1], kn[:, :1], cs, kc, kc, n_sink, window), "Hkv")
    k = torch.zeros(T, Hkv, D, dtype=bf)
    cu = torch.tensor([0, 10, 30, 30, 50, 64], dtype=i32)
    _refused(lambda: S.cache_fill(k, k, cu.long(), kc, kc, n_sink, window), "int32")
    _refused(lambda: S.cache_fill(k, k, cu[:3], kc, kc, n_sink, window), "expected")
