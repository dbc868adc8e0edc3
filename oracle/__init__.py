"""Float64 CPU oracle for learnable-sink attention (ctypes shim).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The CUDA library and
its Python binding never do; the two implementations share no code.

The arithmetic lives in ``sinkattn_oracle.c`` (plain C, float64, OpenMP over
rows), which follows the page "Attention Sink, Learnable Sink and dsink"
(notes.kuangjux.top): the forward of section 4 with the sink as an explicit
extra softmax column, the backward as the explicit Jacobian of that augmented
softmax (sections 7-8), the visible set of section 2, and the StreamingLLM
ring-buffer KV set (sink segment + sliding window).  The gate statistics of
the page "Attention Sink and the native MoE in attention layers"
(lvdousha26.github.io, sections 4-5: head importance and the sink-aware
balance loss) are plain numpy on top of the forward's sink_s.

Every function takes and returns numpy arrays; floating-point inputs are
converted to float64 here (the caller passes the same rounded values the GPU
sees).  The mask is given as plain keyword arguments:
``causal, n_sink, window, cu_seqlens, block_indices, block_q, block_k``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sinkattn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsinkattn_oracle.so")
_lock = threading.Lock()
_lib = None

_d = ctypes.POINTER(ctypes.c_double)
_i32 = ctypes.POINTER(ctypes.c_int32)
_u8 = ctypes.POINTER(ctypes.c_uint8)
_PROBLEM = [ctypes.c_int] * 4 + [ctypes.c_double] + [ctypes.c_int] * 3 + [
    _i32, ctypes.c_int, ctypes.c_int, _i32, ctypes.c_int, ctypes.c_int, ctypes.c_int]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            lib.oracle_fwd.argtypes = _PROBLEM + [_d, _d, _d, _d, _d, _d, _d]
            lib.oracle_fwd_rows.argtypes = _PROBLEM + [
                _d, _d, _d, _d, ctypes.c_int, _i32, _d, _d, _d]
            lib.oracle_bwd.argtypes = _PROBLEM + [_d, _d, _d, _d, _d, _d, _d, _d, _d, _d]
            lib.oracle_bwd_sampled.argtypes = _PROBLEM + [
                _d, _d, _d, _d, _d, ctypes.c_int, _i32, _d, ctypes.c_int, _i32, _d, _d]
            lib.oracle_decode.argtypes = [ctypes.c_int] * 4 + [ctypes.c_double] + [
                _d, _d, _d, _i32, ctypes.c_int, ctypes.c_int, _d, _d, _d, _d]
            lib.oracle_visible_dense.argtypes = _PROBLEM + [ctypes.c_int, _u8]
            lib.oracle_tile_states.argtypes = _PROBLEM + [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, _u8]
            lib.oracle_num_threads.argtypes = []
            _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32arr(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a, typ):
    return None if a is None else a.ctypes.data_as(typ)


class _Problem:
    """Shapes and mask fields in the order the C functions take them."""

    def __init__(self, T_tot, Hq, Hkv, D, scale, causal=True, n_sink=0, window=0,
                 cu_seqlens=None, block_indices=None, block_q=64, block_k=64):
        self.cu = _i32arr(cu_seqlens)
        if self.cu is None:
            self.cu = np.array([0, T_tot], dtype=np.int32)
        self.n_seq = len(self.cu) - 1
        self.bi = _i32arr(block_indices)
        self.max_blocks = 0 if self.bi is None else int(self.bi.shape[-1])
        self.args = (int(T_tot), int(Hq), int(Hkv), int(D), float(scale),
                     int(bool(causal)), int(n_sink), int(window),
                     _p(self.cu, _i32), self.n_seq, 0, _p(self.bi, _i32),
                     int(block_q), int(block_k), self.max_blocks)


def _shapes(q, k):
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    return T, Hq, Hkv, D


def fwd(q, k, v, sink, scale, **mask):
    """Returns (out [T,Hq,D], lse_new [T,Hq], sink_s [T,Hq]) in float64."""
    q, k, v, sink = _f64(q), _f64(k), _f64(v), _f64(sink)
    T, Hq, Hkv, D = _shapes(q, k)
    pr = _Problem(T, Hq, Hkv, D, scale, **mask)
    out = np.zeros((T, Hq, D)); lse = np.zeros((T, Hq)); ss = np.zeros((T, Hq))
    _load().oracle_fwd(*pr.args, _p(q, _d), _p(k, _d), _p(v, _d), _p(sink, _d),
                       _p(out, _d), _p(lse, _d), _p(ss, _d))
    return out, lse, ss


def fwd_rows(q, k, v, sink, scale, rows, **mask):
    """Forward of selected (token, head) rows: rows int array [n, 2].
    Returns (out [n,D], lse [n], sink_s [n])."""
    q, k, v, sink = _f64(q), _f64(k), _f64(v), _f64(sink)
    T, Hq, Hkv, D = _shapes(q, k)
    rows = _i32arr(rows).reshape(-1, 2)
    n = rows.shape[0]
    pr = _Problem(T, Hq, Hkv, D, scale, **mask)
    out = np.zeros((n, D)); lse = np.zeros(n); ss = np.zeros(n)
    _load().oracle_fwd_rows(*pr.args, _p(q, _d), _p(k, _d), _p(v, _d), _p(sink, _d),
                            n, _p(rows, _i32), _p(out, _d), _p(lse, _d), _p(ss, _d))
    return out, lse, ss


def bwd(q, k, v, sink, dout, scale, dss=None, **mask):
    """Returns (dq, dk, dv, dsink) in float64; dsink is None without a sink.
    ``dss`` [T, Hq] is an optional upstream gradient of sink_s (the loss is
    sum dout*O + sum dss*sink_s)."""
    q, k, v, sink, dout, dss = _f64(q), _f64(k), _f64(v), _f64(sink), _f64(dout), _f64(dss)
    T, Hq, Hkv, D = _shapes(q, k)
    pr = _Problem(T, Hq, Hkv, D, scale, **mask)
    dq = np.zeros((T, Hq, D)); dk = np.zeros((T, Hkv, D)); dv = np.zeros((T, Hkv, D))
    dsink = np.zeros(Hq) if sink is not None else None
    rc = _load().oracle_bwd(*pr.args, _p(q, _d), _p(k, _d), _p(v, _d), _p(sink, _d),
                            _p(dout, _d), _p(dss, _d), _p(dq, _d), _p(dk, _d), _p(dv, _d),
                            _p(dsink, _d))
    if rc != 0:
        raise MemoryError("oracle_bwd: allocation failed")
    return dq, dk, dv, dsink


def bwd_sampled(q, k, v, sink, dout, scale, rows, keys, **mask):
    """Gradients on samples of a problem: dQ of rows [(token, head), ...] and
    dK / dV of keys [(token, kv_head), ...].  Returns (dq [n_rows, D],
    dk [n_keys, D], dv [n_keys, D]) in float64."""
    q, k, v, sink, dout = _f64(q), _f64(k), _f64(v), _f64(sink), _f64(dout)
    T, Hq, Hkv, D = _shapes(q, k)
    rows = _i32arr(rows).reshape(-1, 2)
    keys = _i32arr(keys).reshape(-1, 2)
    pr = _Problem(T, Hq, Hkv, D, scale, **mask)
    dq = np.zeros((rows.shape[0], D)); dk = np.zeros((keys.shape[0], D)); dv = np.zeros((keys.shape[0], D))
    rc = _load().oracle_bwd_sampled(*pr.args, _p(q, _d), _p(k, _d), _p(v, _d), _p(sink, _d),
                                    _p(dout, _d), rows.shape[0], _p(rows, _i32), _p(dq, _d),
                                    keys.shape[0], _p(keys, _i32), _p(dk, _d), _p(dv, _d))
    if rc != 0:
        raise MemoryError("oracle_bwd_sampled: allocation failed")
    return dq, dk, dv


def gate_importance(sink_s):
    """Imp_h: the mean gate of head h over every token (page "Attention Sink
    and the native MoE in attention layers", section 4; the gate
    sigma(LSE - sink) of its section 5 is sink_s).  sink_s [T, Hq] -> [Hq]."""
    ss = _f64(sink_s)
    return ss.sum(axis=0) / ss.shape[0]


def gate_aux_loss(imp, lam=1.0, n_shared=0):
    """Sink-aware balance loss of one layer and its gradient d loss / d Imp
    (same page, section 5): lam * (N_h - m) * CV(Imp over routed heads)^2,
    where the m = n_shared heads of largest Imp are shared heads and left out
    (m = 0 is the from-scratch form lam * N_h * CV^2).  CV = std / mean with
    the population standard deviation.  Shared heads get gradient 0 (their
    selection is piecewise constant).  Returns (loss, d_imp [Hq])."""
    imp = _f64(imp)
    n = imp.shape[0]
    order = np.argsort(-imp, kind="stable")
    routed = np.ones(n, dtype=bool)
    routed[order[:n_shared]] = False
    x = imp[routed]
    nr = x.shape[0]
    mu = x.mean()
    var = ((x - mu) ** 2).mean()
    loss = lam * nr * var / mu ** 2
    # d var / d x_i = 2 (x_i - mu) / nr ; d mu / d x_i = 1 / nr
    dx = lam * nr * (2.0 * (x - mu) / nr / mu ** 2 - 2.0 * var / mu ** 3 / nr)
    d_imp = np.zeros(n)
    d_imp[routed] = dx
    return float(loss), d_imp


def gate_vanilla(q, k, scale, **mask):
    """Gate of a sink-free model whose sink is the first token of each
    sequence (page "Attention Sink and the native MoE in attention layers",
    section 5): G = sigma(LSE_not0 - x_0) with x_0 = scale <q, k_0> and LSE_not0
    the log-sum-exp of the visible keys other than k_0.  Readings: a row that
    does not see k_0 puts no mass on it (G = 1); a row that sees no key gets
    G = 0.  Brute force over the visible set.  Returns [T, Hq] float64."""
    q, k = _f64(q), _f64(k)
    T, Hq, Hkv, D = _shapes(q, k)
    G = Hq // Hkv
    cu = _Problem(T, Hq, Hkv, D, scale, **mask).cu
    vis = [visible_dense(T, Hq, Hkv, g, **mask) for g in range(Hkv)]
    out = np.zeros((T, Hq))
    with np.errstate(over="ignore"):
        for s in range(len(cu) - 1):
            j0 = int(cu[s])
            for i in range(int(cu[s]), int(cu[s + 1])):
                for h in range(Hq):
                    keys = np.nonzero(vis[h // G][i])[0]
                    if keys.size == 0:
                        continue
                    if j0 not in keys:
                        out[i, h] = 1.0
                        continue
                    x = scale * (k[keys, h // G] @ q[i, h])
                    x0 = x[keys == j0][0]
                    rest = x[keys != j0]
                    if rest.size == 0:
                        continue  # only k_0 is seen: all mass on it
                    m = rest.max()
                    lse_not0 = m + np.log(np.exp(rest - m).sum())
                    out[i, h] = 1.0 / (1.0 + np.exp(-(lse_not0 - x0)))
    return out


def decode(q, k_cache, v_cache, cache_seqlens, n_sink, window, sink, scale):
    """Ring-buffer decode. q [B,Hq,D], caches [B,S,Hkv,D] (S = n_sink+window).
    Returns (out [B,Hq,D], lse_new [B,Hq], sink_s [B,Hq])."""
    q, kc, vc, sink = _f64(q), _f64(k_cache), _f64(v_cache), _f64(sink)
    cs = _i32arr(cache_seqlens)
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    out = np.zeros((B, Hq, D)); lse = np.zeros((B, Hq)); ss = np.zeros((B, Hq))
    _load().oracle_decode(B, Hq, Hkv, D, float(scale), _p(q, _d), _p(kc, _d),
                          _p(vc, _d), _p(cs, _i32), int(n_sink), int(window),
                          _p(sink, _d), _p(out, _d), _p(lse, _d), _p(ss, _d))
    return out, lse, ss


def fp8_e4m3_value(codes):
    """Value of each FP8 E4M3 code (the OCP 8-bit format without infinities):
    sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
    is subnormal (m / 8 * 2^-6); S.1111.111 is NaN.  uint8 codes -> float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def fp8_e4m3_encode(x):
    """E4M3 code of each value (float32 or float64 array): the nearest value
    of the format's grid (fp8_e4m3_value), ties to the code with an even
    mantissa, magnitudes beyond the largest finite value (448) saturated to
    it, NaN -> the NaN code 0x7F; the sign bit carries the sign (-0.0 and
    negative values that round to zero give 0x80).  Found by search over the
    127 non-negative finite codes, whose values increase with the code."""
    x = np.asarray(x, dtype=np.float64)
    grid = fp8_e4m3_value(np.arange(0x7F, dtype=np.uint8))  # codes 0x00..0x7E, ascending
    a = np.abs(x)
    hi = np.clip(np.searchsorted(grid, a, side="left"), 1, len(grid) - 1)  # grid[hi-1] < a <= grid[hi]
    lo = hi - 1
    d_lo, d_hi = a - grid[lo], grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a <= 0.0, 0, code)
    code = np.where(a >= grid[-1], 0x7E, code)  # saturate
    code = code | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def cache_append_fp8(k_new, v_new, cache_seqlens, k_sink, v_sink, k_win, v_win, k_scale,
                     v_scale, n_sink, window):
    """Mixed-precision ring-cache append (page "Attention Sink / StreamingLLM":
    a fixed sink segment kept in high precision, the sliding window stored
    low).  The token at position p = cache_seqlens[b] - 1 goes to sink slot p
    (copied) if p < n_sink, else to window row (p - n_sink) mod window as E4M3
    codes of value / scale (scale of its KV head; the division in float32, as
    the values and scales are float32).  Returns new copies of the four
    caches (k_sink, v_sink bf16-valued float64 arrays; k_win, v_win uint8)."""
    ks, vs = _f64(k_sink).copy(), _f64(v_sink).copy()
    kw, vw = _u8arr(k_win).copy(), _u8arr(v_win).copy()
    kn, vn = np.asarray(_f64(k_new), dtype=np.float32), np.asarray(_f64(v_new), dtype=np.float32)
    ksc = np.asarray(_f64(k_scale), dtype=np.float32)
    vsc = np.asarray(_f64(v_scale), dtype=np.float32)
    cs = np.asarray(cache_seqlens).astype(np.int64).reshape(-1)
    for b, n in enumerate(cs):
        pos = int(n) - 1
        if pos < 0:
            continue
        if pos < n_sink:
            ks[b, pos] = kn[b]
            vs[b, pos] = vn[b]
        elif window > 0:
            r = (pos - n_sink) % window
            kw[b, r] = fp8_e4m3_encode((kn[b] / ksc[:, None]).astype(np.float32))
            vw[b, r] = fp8_e4m3_encode((vn[b] / vsc[:, None]).astype(np.float32))
    return ks, vs, kw, vw


def decode_fp8_window(q, k_sink, v_sink, k_win, v_win, k_scale, v_scale, cache_seqlens,
                      n_sink, window, sink, scale):
    """Ring-buffer decode with a mixed-precision cache (page "Attention Sink /
    StreamingLLM", on KV-cache quantisation: the first tokens carry much of
    the attention weight, so they stay in high precision and the rest are
    stored low).  k_sink/v_sink [B, n_sink, Hkv, D] hold the sink slots as
    they are; k_win/v_win [B, window, Hkv, D] hold the window slots as FP8
    E4M3 codes whose value is multiplied by a per-KV-head scale
    (k_scale/v_scale [Hkv]).  The cache is dequantised and the float64 decode
    above runs on it.  Returns (out, lse_new, sink_s)."""
    k_scale, v_scale = _f64(k_scale), _f64(v_scale)
    kw = fp8_e4m3_value(_u8arr(k_win)) * k_scale[None, None, :, None]
    vw = fp8_e4m3_value(_u8arr(v_win)) * v_scale[None, None, :, None]
    k = np.concatenate([_f64(k_sink), kw], axis=1)
    v = np.concatenate([_f64(v_sink), vw], axis=1)
    return decode(q, k, v, cache_seqlens, n_sink, window, sink, scale)


def _u8arr(x):
    """uint8 codes from a numpy array or a torch tensor of any 1-byte type."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().cpu().contiguous().view(torch.uint8).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint8))


def visible_dense(T_tot, Hq, Hkv, g, **mask):
    """Dense visibility matrix [T, T] (uint8) of KV head g."""
    pr = _Problem(T_tot, Hq, Hkv, 1, 1.0, **mask)
    vis = np.zeros((T_tot, T_tot), dtype=np.uint8)
    _load().oracle_visible_dense(*pr.args, int(g), _p(vis, _u8))
    return vis


def tile_states(T_tot, Hq, Hkv, tile_q, tile_k, **mask):
    """Brute-force tile classification: uint8 [Hkv, n_qtiles, max_ktiles]
    with 0 = no visible pair, 1 = partly visible, 2 = fully visible."""
    pr = _Problem(T_tot, Hq, Hkv, 1, 1.0, **mask)
    lens = np.diff(pr.cu)
    nqt = int(sum((int(l) + tile_q - 1) // tile_q for l in lens))
    max_kt = int((int(lens.max()) + tile_k - 1) // tile_k) if len(lens) else 0
    st = np.zeros((Hkv, max(nqt, 1), max(max_kt, 1)), dtype=np.uint8)
    _load().oracle_tile_states(*pr.args, int(tile_q), int(tile_k), max(max_kt, 1),
                               _p(st, _u8))
    return st[:, :nqt, :max_kt]
