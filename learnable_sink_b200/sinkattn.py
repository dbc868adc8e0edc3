"""Thin Python binding of libsinkattn.so (ctypes; argument marshalling only).

Every computation runs in the CUDA library; this module only checks tensor
metadata, allocates outputs with torch, and passes raw device pointers and
the current CUDA stream through the C ABI declared in ``include/sinkattn.h``.
There is no fallback: if the library is missing or the device is not a B200
(sm_100a), calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsinkattn.so")

BF16, FP16, FP32 = 0, 1, 2
OK = 0
ERR_NAMES = {1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "WORKSPACE", 5: "TIMEOUT",
             6: "BOUNDS", 7: "PLAN"}

_c = ctypes
_vp = _c.c_void_p
_i = _c.c_int
_sz = _c.c_size_t


class CMask(_c.Structure):
    """Mirror of ``sinkattn_mask``."""
    _fields_ = [("causal", _c.c_int32), ("n_sink", _c.c_int32), ("window", _c.c_int32),
                ("cu_seqlens", _vp), ("n_seq", _c.c_int32), ("max_seqlen", _c.c_int32),
                ("block_indices", _vp), ("n_qblk", _c.c_int32), ("block_q", _c.c_int32),
                ("block_k", _c.c_int32), ("max_blocks", _c.c_int32)]


class SinkAttnError(RuntimeError):
    def __init__(self, fn, code, detail=None):
        msg = f"{fn} failed: {ERR_NAMES.get(code, code)} ({error_string(code)})"
        super().__init__(msg if detail is None else f"{msg}: {detail}")
        self.code = code


_lib = None


def lib():
    """Load libsinkattn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m learnable_sink_b200.build` (nvcc, sm_100a)")
        L = _c.CDLL(LIB_PATH)
        M = _c.POINTER(CMask)
        L.sinkattn_plan_bytes.restype = _sz
        L.sinkattn_plan_bytes.argtypes = [_i, _i, _i, M]
        L.sinkattn_plan.argtypes = [_i, _i, _i, M, _vp, _sz, _vp]
        L.sinkattn_fwd.argtypes = [_i, _i, _i, _i, _i, _c.c_float, _vp, _vp, _vp, _vp, M, _vp, _sz,
                                   _vp, _vp, _vp, _vp]
        L.sinkattn_fwd_ex.argtypes = [_i, _i, _i, _i, _i, _c.c_float, _vp, _vp, _vp, _vp, M, _vp,
                                      _sz, _vp, _vp, _vp, _vp, _vp]
        L.sinkattn_bwd_workspace_bytes.restype = _sz
        L.sinkattn_bwd_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, M]
        L.sinkattn_bwd.argtypes = [_i, _i, _i, _i, _i, _c.c_float, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, M, _vp, _sz, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
        L.sinkattn_bwd_ex.argtypes = [_i, _i, _i, _i, _i, _c.c_float, _vp, _vp, _vp, _vp, _vp,
                                      _vp, _vp, _vp, M, _vp, _sz, _vp, _vp, _vp, _vp, _vp, _sz,
                                      _vp]
        L.sinkattn_gate_importance_workspace_bytes.restype = _sz
        L.sinkattn_gate_importance_workspace_bytes.argtypes = [_i, _i]
        L.sinkattn_gate_importance.argtypes = [_i, _i, _vp, _vp, _vp, _sz, _vp]
        L.sinkattn_gate_vanilla.argtypes = [_i, _i, _i, _i, _i, _c.c_float, _vp, _vp, _vp, M,
                                            _vp, _vp]
        L.sinkattn_decode_workspace_bytes.restype = _sz
        L.sinkattn_decode_workspace_bytes.argtypes = [_i, _i, _i, _i]
        L.sinkattn_decode_num_splits.argtypes = [_i, _i, _i, _i, _i, _i]
        L.sinkattn_decode.argtypes = [_i, _i, _i, _i, _i, _c.c_float, _vp, _vp, _vp, _vp, _i, _i,
                                      _vp, _vp, _vp, _vp, _i, _vp, _sz, _vp]
        L.sinkattn_decode_fp8_num_splits.argtypes = [_i, _i, _i, _i, _i, _i]
        L.sinkattn_decode_fp8.argtypes = [_i, _i, _i, _i, _c.c_float, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp, _vp, _i, _i, _vp, _vp, _vp, _vp, _i, _vp,
                                          _sz, _vp]
        L.sinkattn_cache_append_fp8.argtypes = [_i, _i, _i, _i, _i] + [_vp] * 9 + [_vp]
        L.sinkattn_cache_append.argtypes = [_i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]
        L.sinkattn_cache_fill.argtypes = [_i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                                          _vp, _vp]
        L.sinkattn_set_kernel_events.argtypes = [_i, _vp, _vp]
        L.sinkattn_selftest_timeout.argtypes = [_vp]
        L.sinkattn_get_status.argtypes = [_vp]
        L.sinkattn_clear_status.argtypes = [_vp]
        L.sinkattn_error_string.restype = _c.c_char_p
        L.sinkattn_error_string.argtypes = [_i]
        L.sinkattn_version.argtypes = []
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().sinkattn_error_string(code).decode()


def _check(fn, code):
    if code != OK:
        raise SinkAttnError(fn, code)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else _vp(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return _vp(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return FP16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16, float16 or float32")


@dataclass
class Mask:
    """Mask descriptor.  ``cu_seqlens`` / ``block_indices`` are int32 CUDA
    tensors; ``max_seqlen`` must bound every sequence length."""
    cu_seqlens: torch.Tensor
    max_seqlen: int
    causal: bool = True
    n_sink: int = 0
    window: int = 0
    block_indices: Optional[torch.Tensor] = None
    block_q: int = 64
    block_k: int = 64

    def c(self) -> CMask:
        bi = self.block_indices
        return CMask(int(bool(self.causal)), int(self.n_sink), int(self.window),
                     self.cu_seqlens.data_ptr(), int(self.cu_seqlens.numel() - 1),
                     int(self.max_seqlen), None if bi is None else bi.data_ptr(),
                     0 if bi is None else int(bi.shape[1]), int(self.block_q), int(self.block_k),
                     0 if bi is None else int(bi.shape[2]))

    @staticmethod
    def from_spec(spec, device="cuda") -> "Mask":
        """From :class:`learnable_sink_b200.workloads.MaskSpec` (CPU tensors)."""
        bi = spec.block_indices
        return Mask(cu_seqlens=spec.cu_seqlens.to(device=device, dtype=torch.int32).contiguous(),
                    max_seqlen=max(1, spec.max_seqlen), causal=spec.causal, n_sink=spec.n_sink,
                    window=spec.window,
                    block_indices=None if bi is None else bi.to(device=device, dtype=torch.int32).contiguous(),
                    block_q=spec.block_q, block_k=spec.block_k)


class Plan:
    """Tile schedule built on the device from a mask (reusable by fwd/bwd)."""

    def __init__(self, T_tot: int, Hq: int, Hkv: int, mask: Mask, stream=None):
        self.T_tot, self.Hq, self.Hkv, self.mask = T_tot, Hq, Hkv, mask
        self._cm = mask.c()
        nbytes = lib().sinkattn_plan_bytes(T_tot, Hq, Hkv, _c.byref(self._cm))
        if nbytes == 0:
            raise SinkAttnError("sinkattn_plan_bytes", 1)
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=mask.cu_seqlens.device)
        self.rebuild(stream)

    def rebuild(self, stream=None) -> None:
        """Rebuild the schedule in place (e.g. after the mask arrays changed)."""
        _check("sinkattn_plan", lib().sinkattn_plan(self.T_tot, self.Hq, self.Hkv,
                                                    _c.byref(self._cm), _ptr(self.buf),
                                                    self.buf.numel(), _stream(stream)))

    @property
    def nbytes(self) -> int:
        return self.buf.numel()


def _want(fn, ok, detail):
    """Metadata the C ABI cannot see through raw pointers (element types and
    extents); a mismatch would make a kernel read or write outside a buffer,
    so it is refused here as SINKATTN_ERR_INVALID_ARG before any launch."""
    if not ok:
        raise SinkAttnError(fn, 1, detail)


def _same_type(fn, ref, **ts):
    for name, t in ts.items():
        if t is not None:
            _want(fn, t.dtype == ref.dtype, f"{name} is {t.dtype}, expected {ref.dtype}")


def _shape(fn, name, t, shape, dtype=None):
    if t is None:
        return
    _want(fn, tuple(t.shape) == tuple(shape),
          f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None:
        _want(fn, t.dtype == dtype, f"{name} is {t.dtype}, expected {dtype}")


def _attn_meta(fn, q, k, v, mask):
    _want(fn, q.dim() == 3 and k.dim() == 3 and v.dim() == 3, "q, k, v must be [T, H, D]")
    _same_type(fn, q, k=k, v=v)
    _want(fn, tuple(k.shape) == tuple(v.shape), "k and v shapes differ")
    _want(fn, q.shape[0] == k.shape[0] and q.shape[2] == k.shape[2],
          f"q {tuple(q.shape)} and k {tuple(k.shape)} disagree on T or D")
    _want(fn, mask.cu_seqlens.dtype == torch.int32, "cu_seqlens must be int32")
    if mask.block_indices is not None:
        _want(fn, mask.block_indices.dtype == torch.int32, "block_indices must be int32")


def _ring_meta(fn, k_cache, v_cache, ref, B, D, n_sink, window):
    _same_type(fn, ref, k_cache=k_cache, v_cache=v_cache)
    _want(fn, tuple(k_cache.shape) == tuple(v_cache.shape), "k_cache and v_cache shapes differ")
    S_ = int(n_sink) + int(window)
    _want(fn, k_cache.shape[0] == B and k_cache.shape[1] == S_ and k_cache.shape[3] == D,
          f"caches have shape {tuple(k_cache.shape)}, expected [{B}, n_sink + window = {S_}, "
          f"Hkv, {D}]")


def _contig(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def fwd(q, k, v, sink, mask: Mask, plan: Plan, scale: Optional[float] = None, stream=None,
        out=None, lse=None, sink_s=None, lse_orig=None):
    """Forward.  Returns (out [T,Hq,D], lse_new [T,Hq] fp32, sink_s [T,Hq] fp32).
    With ``lse_orig`` (fp32 [T,Hq]) also writes the LSE over the visible keys
    alone, before the sink joins (sinkattn_fwd_ex)."""
    _attn_meta("sinkattn_fwd", q, k, v, mask)
    T, Hq, D = q.shape
    _shape("sinkattn_fwd", "learnable_sink", sink, (Hq,), torch.float32)
    _shape("sinkattn_fwd", "out", out, q.shape, q.dtype)
    for name, t in (("lse", lse), ("sink_s", sink_s), ("lse_orig", lse_orig)):
        _shape("sinkattn_fwd", name, t, (T, Hq), torch.float32)
    _contig(q, k, v, sink)
    Hkv = k.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(T, Hq, dtype=torch.float32, device=q.device) if lse is None else lse
    sink_s = torch.empty(T, Hq, dtype=torch.float32, device=q.device) if sink_s is None else sink_s
    cm = mask.c()
    if lse_orig is None:
        _check("sinkattn_fwd", lib().sinkattn_fwd(
            _dt(q), T, Hq, Hkv, D, scale, _ptr(q), _ptr(k), _ptr(v), _ptr(sink), _c.byref(cm),
            _ptr(plan.buf), plan.nbytes, _ptr(out), _ptr(lse), _ptr(sink_s), _stream(stream)))
    else:
        _contig(lse_orig)
        _check("sinkattn_fwd_ex", lib().sinkattn_fwd_ex(
            _dt(q), T, Hq, Hkv, D, scale, _ptr(q), _ptr(k), _ptr(v), _ptr(sink), _c.byref(cm),
            _ptr(plan.buf), plan.nbytes, _ptr(out), _ptr(lse), _ptr(sink_s), _ptr(lse_orig),
            _stream(stream)))
    return out, lse, sink_s


def bwd_workspace_bytes(q, k, mask: Mask) -> int:
    T, Hq, D = q.shape
    cm = mask.c()
    return int(lib().sinkattn_bwd_workspace_bytes(_dt(q), T, Hq, k.shape[1], D, _c.byref(cm)))


def bwd(q, k, v, out, dout, lse, sink, mask: Mask, plan: Plan, scale: Optional[float] = None,
        stream=None, workspace=None, dq=None, dk=None, dv=None, dsink=None, d_sink_s=None):
    """Backward.  Returns (dq, dk, dv, dsink or None).  ``d_sink_s`` [T, Hq]
    float32 is an optional upstream gradient of the gate sink_s."""
    _attn_meta("sinkattn_bwd", q, k, v, mask)
    T, Hq, D = q.shape
    _same_type("sinkattn_bwd", q, out=out, dout=dout, dq=dq, dk=dk, dv=dv)
    for name, t in (("out", out), ("dout", dout), ("dq", dq)):
        _shape("sinkattn_bwd", name, t, q.shape)
    for name, t in (("dk", dk), ("dv", dv)):
        _shape("sinkattn_bwd", name, t, k.shape)
    for name, t in (("lse", lse), ("d_sink_s", d_sink_s)):
        _shape("sinkattn_bwd", name, t, (T, Hq), torch.float32)
    for name, t in (("learnable_sink", sink), ("dsink", dsink)):
        _shape("sinkattn_bwd", name, t, (Hq,), torch.float32)
    _contig(q, k, v, out, dout, lse, sink, d_sink_s)
    Hkv = k.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    cm = mask.c()
    nws = lib().sinkattn_bwd_workspace_bytes(_dt(q), T, Hq, Hkv, D, _c.byref(cm))
    if workspace is None:
        workspace = torch.empty(max(nws, 16), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if dsink is None and sink is not None:
        dsink = torch.empty(Hq, dtype=torch.float32, device=q.device)
    _check("sinkattn_bwd_ex", lib().sinkattn_bwd_ex(
        _dt(q), T, Hq, Hkv, D, scale, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
        _ptr(d_sink_s), _ptr(sink), _c.byref(cm), _ptr(plan.buf), plan.nbytes, _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(dsink), _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv, dsink


def gate_importance(sink_s, stream=None, workspace=None, imp=None):
    """Per-head mean gate Imp [Hq] of sink_s [T, Hq] float32."""
    _want("sinkattn_gate_importance", sink_s.dim() == 2 and sink_s.dtype == torch.float32,
          "sink_s must be float32 [T, Hq]")
    T, Hq = sink_s.shape
    _shape("sinkattn_gate_importance", "imp", imp, (Hq,), torch.float32)
    _contig(sink_s)
    nws = int(lib().sinkattn_gate_importance_workspace_bytes(T, Hq))
    if workspace is None:
        workspace = torch.empty(max(nws, 16), dtype=torch.uint8, device=sink_s.device)
    imp = torch.empty(Hq, dtype=torch.float32, device=sink_s.device) if imp is None else imp
    _check("sinkattn_gate_importance", lib().sinkattn_gate_importance(
        T, Hq, _ptr(sink_s), _ptr(imp), _ptr(workspace), workspace.numel(), _stream(stream)))
    return imp


def gate_vanilla(q, k, lse, mask: Mask, scale: Optional[float] = None, stream=None, gate=None):
    """Gate sigma(LSE_not0 - q.k_0 scale) [T, Hq] of a sink-free model whose
    sink is each sequence's first token; ``lse`` is the sink-free LSE."""
    _attn_meta("sinkattn_gate_vanilla", q, k, k, mask)
    T, Hq, D = q.shape
    for name, t in (("lse", lse), ("gate", gate)):
        _shape("sinkattn_gate_vanilla", name, t, (T, Hq), torch.float32)
    _contig(q, k, lse, gate)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    cm = mask.c()
    gate = torch.empty(T, Hq, dtype=torch.float32, device=q.device) if gate is None else gate
    _check("sinkattn_gate_vanilla", lib().sinkattn_gate_vanilla(
        _dt(q), T, Hq, k.shape[1], D, scale, _ptr(q), _ptr(k), _ptr(lse), _c.byref(cm),
        _ptr(gate), _stream(stream)))
    return gate


def decode_num_splits(B, Hq, Hkv, D, n_sink, window) -> int:
    return int(lib().sinkattn_decode_num_splits(B, Hq, Hkv, D, n_sink, window))


def decode_workspace_bytes(B, Hq, D, num_splits) -> int:
    return int(lib().sinkattn_decode_workspace_bytes(B, Hq, D, num_splits))


def decode(q, k_cache, v_cache, cache_seqlens, n_sink: int, window: int, sink,
           scale: Optional[float] = None, num_splits: int = 0, stream=None, workspace=None,
           out=None, lse=None, sink_s=None):
    """Ring-buffer decode.  Returns (out [B,Hq,D], lse_new [B,Hq], sink_s [B,Hq])."""
    fn = "sinkattn_decode"
    _want(fn, q.dim() == 3 and k_cache.dim() == 4, "q must be [B, Hq, D], caches [B, S, Hkv, D]")
    B, Hq, D = q.shape
    _ring_meta(fn, k_cache, v_cache, q, B, D, n_sink, window)
    _shape(fn, "cache_seqlens", cache_seqlens, (B,), torch.int32)
    _shape(fn, "learnable_sink", sink, (Hq,), torch.float32)
    _shape(fn, "out", out, q.shape, q.dtype)
    for name, t in (("lse", lse), ("sink_s", sink_s)):
        _shape(fn, name, t, (B, Hq), torch.float32)
    _contig(q, k_cache, v_cache, cache_seqlens, sink)
    Hkv = k_cache.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if num_splits <= 0:
        num_splits = decode_num_splits(B, Hq, Hkv, D, n_sink, window)
    nws = decode_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None:
        workspace = torch.empty(max(nws, 16), dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device) if lse is None else lse
    sink_s = torch.empty(B, Hq, dtype=torch.float32, device=q.device) if sink_s is None else sink_s
    _check("sinkattn_decode", lib().sinkattn_decode(
        _dt(q), B, Hq, Hkv, D, scale, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens),
        int(n_sink), int(window), _ptr(sink), _ptr(out), _ptr(lse), _ptr(sink_s), int(num_splits),
        _ptr(workspace), workspace.numel(), _stream(stream)))
    return out, lse, sink_s


def decode_fp8_num_splits(B, Hq, Hkv, D, n_sink, window) -> int:
    return int(lib().sinkattn_decode_fp8_num_splits(B, Hq, Hkv, D, n_sink, window))


def decode_fp8(q, k_sink, v_sink, k_win, v_win, k_scale, v_scale, cache_seqlens, n_sink: int,
               window: int, sink, scale: Optional[float] = None, num_splits: int = 0,
               stream=None, workspace=None, out=None, lse=None, sink_s=None):
    """Ring-buffer decode over a mixed-precision cache: bf16 sink slots
    k_sink/v_sink [B, n_sink, Hkv, D], FP8 E4M3 window slots k_win/v_win
    [B, window, Hkv, D] (uint8 codes, or torch.float8_e4m3fn) with per-KV-head
    float32 scales k_scale/v_scale [Hkv].  Returns (out [B,Hq,D] bf16,
    lse_new [B,Hq], sink_s [B,Hq])."""
    fn = "sinkattn_decode_fp8"
    _want(fn, q.dim() == 3 and q.dtype == torch.bfloat16, "q must be bfloat16 [B, Hq, D]")
    B, Hq, D = q.shape
    _want(fn, k_win.dim() == 4 and k_win.element_size() == 1 and v_win.element_size() == 1,
          "k_win / v_win must be 1-byte [B, window, Hkv, D] E4M3 codes")
    Hkv = k_win.shape[2]
    _shape(fn, "k_win", k_win, (B, window, Hkv, D))
    _shape(fn, "v_win", v_win, (B, window, Hkv, D))
    for name, t in (("k_sink", k_sink), ("v_sink", v_sink)):
        _shape(fn, name, t, (B, n_sink, Hkv, D), torch.bfloat16)
    for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
        _shape(fn, name, t, (Hkv,), torch.float32)
    _shape(fn, "cache_seqlens", cache_seqlens, (B,), torch.int32)
    _shape(fn, "learnable_sink", sink, (Hq,), torch.float32)
    _shape(fn, "out", out, q.shape, q.dtype)
    for name, t in (("lse", lse), ("sink_s", sink_s)):
        _shape(fn, name, t, (B, Hq), torch.float32)
    _contig(q, k_sink, v_sink, k_win, v_win, k_scale, v_scale, cache_seqlens, sink)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if num_splits <= 0:
        num_splits = decode_fp8_num_splits(B, Hq, Hkv, D, n_sink, window)
    nws = decode_workspace_bytes(B, Hq, D, num_splits)
    if workspace is None:
        workspace = torch.empty(max(nws, 16), dtype=torch.uint8, device=q.device)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty(B, Hq, dtype=torch.float32, device=q.device) if lse is None else lse
    sink_s = torch.empty(B, Hq, dtype=torch.float32, device=q.device) if sink_s is None else sink_s
    _check(fn, lib().sinkattn_decode_fp8(
        B, Hq, Hkv, D, scale, _ptr(q), _ptr(k_sink), _ptr(v_sink), _ptr(k_win), _ptr(v_win),
        _ptr(k_scale), _ptr(v_scale), _ptr(cache_seqlens), int(n_sink), int(window), _ptr(sink),
        _ptr(out), _ptr(lse), _ptr(sink_s), int(num_splits), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return out, lse, sink_s


def cache_append(k_new, v_new, cache_seqlens, k_cache, v_cache, n_sink: int, window: int,
                 stream=None) -> None:
    """Write one new token per sequence (k_new/v_new [B, Hkv, D]) into its ring
    slot; cache_seqlens [B] int32 already counts the new token."""
    fn = "sinkattn_cache_append"
    _want(fn, k_new.dim() == 3 and k_cache.dim() == 4, "k_new must be [B, Hkv, D]")
    B, Hkv, D = k_new.shape
    _shape(fn, "v_new", v_new, k_new.shape, k_new.dtype)
    _ring_meta(fn, k_cache, v_cache, k_new, B, D, n_sink, window)
    _want(fn, k_cache.shape[2] == Hkv, "k_new and the caches disagree on Hkv")
    _shape(fn, "cache_seqlens", cache_seqlens, (B,), torch.int32)
    _contig(k_new, v_new, cache_seqlens, k_cache, v_cache)
    _check("sinkattn_cache_append", lib().sinkattn_cache_append(
        _dt(k_new), B, Hkv, D, int(n_sink), int(window), _ptr(k_new), _ptr(v_new),
        _ptr(cache_seqlens), _ptr(k_cache), _ptr(v_cache), _stream(stream)))


def cache_append_fp8(k_new, v_new, cache_seqlens, k_sink, v_sink, k_win, v_win, k_scale,
                     v_scale, n_sink: int, window: int, stream=None) -> None:
    """Write one new bf16 token per sequence (k_new/v_new [B, Hkv, D]) into
    the mixed-precision cache of decode_fp8: a sink slot as it is, a window
    row as E4M3 codes of value / scale; cache_seqlens [B] int32 already
    counts the new token."""
    fn = "sinkattn_cache_append_fp8"
    _want(fn, k_new.dim() == 3 and k_new.dtype == torch.bfloat16, "k_new must be bf16 [B, Hkv, D]")
    B, Hkv, D = k_new.shape
    _shape(fn, "v_new", v_new, k_new.shape, k_new.dtype)
    for name, t in (("k_sink", k_sink), ("v_sink", v_sink)):
        _shape(fn, name, t, (B, n_sink, Hkv, D), torch.bfloat16)
    for name, t in (("k_win", k_win), ("v_win", v_win)):
        if t is not None:
            _want(fn, t.element_size() == 1, f"{name} must hold 1-byte E4M3 codes")
        _shape(fn, name, t, (B, window, Hkv, D))
    for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
        _shape(fn, name, t, (Hkv,), torch.float32)
    _shape(fn, "cache_seqlens", cache_seqlens, (B,), torch.int32)
    _contig(k_new, v_new, cache_seqlens, k_sink, v_sink, k_win, v_win, k_scale, v_scale)
    _check(fn, lib().sinkattn_cache_append_fp8(
        B, Hkv, D, int(n_sink), int(window), _ptr(k_new), _ptr(v_new), _ptr(cache_seqlens),
        _ptr(k_sink), _ptr(v_sink), _ptr(k_win), _ptr(v_win), _ptr(k_scale), _ptr(v_scale),
        _stream(stream)))


def cache_fill(k, v, cu_seqlens, k_cache, v_cache, n_sink: int, window: int,
               cache_seqlens_out=None, stream=None) -> None:
    """Write a packed prefill (k/v [T_tot, Hkv, D], sequences by cu_seqlens)
    into the ring caches [n_seq, S, Hkv, D]; optionally store the lengths."""
    fn = "sinkattn_cache_fill"
    _want(fn, k.dim() == 3 and k_cache.dim() == 4 and cu_seqlens.dim() == 1,
          "k must be [T, Hkv, D], caches [n_seq, S, Hkv, D], cu_seqlens [n_seq + 1]")
    T, Hkv, D = k.shape
    n_seq = cu_seqlens.numel() - 1
    _shape(fn, "v", v, k.shape, k.dtype)
    _want(fn, cu_seqlens.dtype == torch.int32, "cu_seqlens must be int32")
    _ring_meta(fn, k_cache, v_cache, k, n_seq, D, n_sink, window)
    _want(fn, k_cache.shape[2] == Hkv, "k and the caches disagree on Hkv")
    _shape(fn, "cache_seqlens_out", cache_seqlens_out, (n_seq,), torch.int32)
    _contig(k, v, cu_seqlens, k_cache, v_cache, cache_seqlens_out)
    n_seq = cu_seqlens.numel() - 1
    _check("sinkattn_cache_fill", lib().sinkattn_cache_fill(
        _dt(k), n_seq, T, Hkv, D, int(n_sink), int(window), _ptr(cu_seqlens), _ptr(k), _ptr(v),
        _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens_out), _stream(stream)))


KERNEL_FWD, KERNEL_BWD, KERNEL_DECODE, KERNEL_GATE = 0, 1, 2, 3


def set_kernel_events(which: int, start=None, stop=None) -> None:
    """Have later calls record torch.cuda.Event ``start``/``stop`` around their
    main kernel (events must already have been recorded once, so that torch
    has created them).  Pass None, None to stop."""
    sp = None if start is None else _vp(start.cuda_event)
    ep = None if stop is None else _vp(stop.cuda_event)
    _check("sinkattn_set_kernel_events", lib().sinkattn_set_kernel_events(int(which), sp, ep))


def selftest_timeout(stream=None) -> None:
    """Launch the bounded-wait self-test kernel (see include/sinkattn.h)."""
    _check("sinkattn_selftest_timeout", lib().sinkattn_selftest_timeout(_stream(stream)))


def get_status(stream=None) -> int:
    return int(lib().sinkattn_get_status(_stream(stream)))


def clear_status(stream=None) -> None:
    _check("sinkattn_clear_status", lib().sinkattn_clear_status(_stream(stream)))
