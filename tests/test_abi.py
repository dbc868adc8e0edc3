"""The C-ABI library loads and exports every symbol include/sinkattn.h
declares; host-only queries behave (no GPU needed, no kernel launched)."""
import ctypes
import os
import re

import pytest

from learnable_sink_b200 import sinkattn as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sinkattn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sinkattn_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(S.LIB_PATH):
        import learnable_sink_b200.build as B
        B.build()
    return S.lib()


def test_header_declares_the_three_entry_points():
    fns = declared_functions()
    for name in ("sinkattn_fwd", "sinkattn_bwd", "sinkattn_decode", "sinkattn_plan"):
        assert name in fns


def test_every_declared_symbol_is_exported(lib):
    missing = [f for f in declared_functions() if not hasattr(lib, f)]
    assert not missing, missing


def test_error_strings_and_version(lib):
    assert S.error_string(0) == "ok"
    for code in range(1, 8):
        assert S.error_string(code) != "unknown error"
    assert lib.sinkattn_version() >= 100


def _mask(**kw):
    m = S.CMask(1, 0, 0, 16, 1, 128, None, 0, 64, 64, 0)  # fake aligned device pointer
    for k, v in kw.items():
        setattr(m, k, v)
    return m


def test_plan_bytes_validates_masks(lib):
    ok = _mask()
    assert lib.sinkattn_plan_bytes(128, 4, 2, ctypes.byref(ok)) > 0
    assert lib.sinkattn_plan_bytes(128, 3, 2, ctypes.byref(ok)) == 0         # Hq % Hkv
    assert lib.sinkattn_plan_bytes(128, 4, 2, ctypes.byref(_mask(causal=0, window=8))) == 0
    assert lib.sinkattn_plan_bytes(128, 4, 2, ctypes.byref(_mask(cu_seqlens=None))) == 0
    assert lib.sinkattn_plan_bytes(128, 4, 2, ctypes.byref(_mask(cu_seqlens=8))) == 0  # misaligned
    bs = _mask(block_indices=32, n_qblk=2, max_blocks=17)
    assert lib.sinkattn_plan_bytes(128, 4, 2, ctypes.byref(bs)) > 0
    assert lib.sinkattn_plan_bytes(128, 4, 2, ctypes.byref(_mask(block_indices=32, n_qblk=2, max_blocks=33))) == 0
    assert lib.sinkattn_plan_bytes(128, 4, 2, ctypes.byref(_mask(block_indices=32, n_qblk=2, max_blocks=4, block_q=32, block_k=32))) == 0


def test_workspace_queries(lib):
    m = _mask()
    assert lib.sinkattn_bwd_workspace_bytes(0, 128, 4, 2, 64, ctypes.byref(m)) >= 128 * 4 * 4
    assert lib.sinkattn_bwd_workspace_bytes(0, 128, 4, 2, 96, ctypes.byref(m)) == 0
    assert lib.sinkattn_decode_workspace_bytes(32, 32, 128, 4) >= 32 * 32 * 4 * 130 * 4
    assert lib.sinkattn_decode_workspace_bytes(32, 32, 80, 4) == 0
    lib.sinkattn_gate_importance_workspace_bytes.restype = ctypes.c_size_t
    # one float64 partial per head per CTA of at least 32 tokens, at most 1024 CTAs
    assert lib.sinkattn_gate_importance_workspace_bytes(100, 32) == 4 * 32 * 8
    assert lib.sinkattn_gate_importance_workspace_bytes(10 ** 6, 8) == 1024 * 8 * 8
    assert lib.sinkattn_gate_importance_workspace_bytes(0, 8) == 0
    assert lib.sinkattn_gate_importance_workspace_bytes(64, 257) == 0


def test_gate_importance_host_validation(lib):
    """Argument checks that return before anything reaches a device."""
    f = lib.sinkattn_gate_importance
    f.argtypes = [ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 3 + [ctypes.c_size_t,
                                                                        ctypes.c_void_p]
    assert f(0, 8, None, None, None, 0, None) == 1      # T_tot < 1
    assert f(16, 0, None, None, None, 0, None) == 1     # Hq < 1
    assert f(16, 257, None, None, None, 0, None) == 2   # more heads than supported
    assert f(16, 8, None, None, None, 0, None) == 1     # null pointers


def test_gate_vanilla_and_bwd_ex_host_validation(lib):
    """Invalid arguments are refused on the host, before any device query."""
    m = _mask()
    a16 = 256  # stand-in 16-byte-aligned device addresses: never dereferenced here
    gv = lib.sinkattn_gate_vanilla
    assert gv(0, 128, 4, 2, 96, 0.1, a16, a16, a16, ctypes.byref(m), a16, None) == 1  # D
    assert gv(3, 128, 4, 2, 64, 0.1, a16, a16, a16, ctypes.byref(m), a16, None) == 1  # no such dtype
    assert gv(0, 128, 4, 2, 64, 0.1, None, a16, a16, ctypes.byref(m), a16, None) == 1  # q
    assert gv(0, 128, 4, 2, 64, 0.1, a16, a16, a16, ctypes.byref(m), None, None) == 1  # gate
    assert gv(0, 128, 4, 2, 64, 0.1, a16 + 8, a16, a16, ctypes.byref(m), a16, None) == 1
    assert gv(0, 128, 3, 2, 64, 0.1, a16, a16, a16, ctypes.byref(m), a16, None) == 1  # Hq % Hkv
    bad = _mask(causal=0, window=8)                                                # window needs causal
    assert gv(0, 128, 4, 2, 64, 0.1, a16, a16, a16, ctypes.byref(bad), a16, None) == 1
    bx = lib.sinkattn_bwd_ex
    args = [a16] * 5 + [a16, None, None]  # q k v out dout lse d_sink_s learnable_sink
    tail = [a16, 1 << 20, a16, a16, a16, None, a16, 1 << 20, None]
    assert bx(0, 128, 4, 2, 96, 0.1, *args, ctypes.byref(m), *tail) == 1   # D
    assert bx(0, 128, 4, 2, 64, 0.1, None, *args[1:], ctypes.byref(m), *tail) == 1  # q


def test_decode_split_heuristic(lib):
    """The fewest partial slots per (sequence, KV head) that still give each
    streaming warp (8 on each of 148 SMs when no device is visible) an equal
    run of 16-row pieces: runs of ppw = ceil(total pieces / warps), and a
    pair of np pieces meets at most ceil((np - 1) / ppw) + 1 runs; never more
    slots than pieces, never more than 128."""
    f = lib.sinkattn_decode_num_splits
    # 256 pairs x 64 pieces over 1184 warps: runs of 14 pieces
    assert f(32, 32, 8, 128, 4, 1020) == 6                 # ceil(63 / 14) + 1
    assert f(1, 32, 8, 128, 4, 1020) == 64                 # runs of 1 piece: one slot per piece
    # 6251 pieces: runs of 50 keep the slots within 128
    assert f(1, 8, 1, 128, 4, 100000) == 126               # ceil(6250 / 50) + 1
    assert f(4096, 64, 8, 128, 4, 1020) == 2               # runs longer than a pair
    assert f(0, 8, 1, 128, 4, 100) == 1                    # degenerate sizes


def test_decode_fp8_host_validation_and_split_heuristic(lib):
    """The mixed-precision decode's host checks refuse bad arguments before any
    device query; its split count follows the same rule over its pieces
    (16-row sink pieces, 32-row window pieces)."""
    f = lib.sinkattn_decode_fp8
    f.argtypes = [ctypes.c_int] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 8 + \
        [ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 4 + [ctypes.c_int, ctypes.c_void_p,
                                                                 ctypes.c_size_t, ctypes.c_void_p]
    a = 256  # stand-in 16-byte-aligned device address: never dereferenced here
    ok = [a] * 8  # q k_sink v_sink k_win v_win k_scale v_scale cache_seqlens

    def call(B=2, Hq=8, Hkv=2, D=128, ptrs=ok, n_sink=4, window=60, out=a, ws=a, ws_bytes=1 << 20):
        return f(B, Hq, Hkv, D, 0.1, *ptrs, n_sink, window, None, out, a, None, 0, ws, ws_bytes,
                 None)

    assert call(D=96) == 1                        # head dimension
    assert call(Hq=6, Hkv=4) == 1                 # Hq % Hkv
    assert call(Hq=32, Hkv=2) == 2                # 16 query heads per KV head: unsupported
    assert call(n_sink=0, window=0) == 1          # empty cache
    assert call(ptrs=[a, None] + ok[2:]) == 1     # sink slots without k_sink
    assert call(ptrs=ok[:3] + [a + 8] + ok[4:]) == 1  # misaligned window codes
    assert call(out=None) == 1
    assert call(ws_bytes=16) == 4                 # workspace too small
    ns = lib.sinkattn_decode_fp8_num_splits
    # 32 x 8 pairs x (1 sink piece + 32 window pieces) over 1184 warps: runs
    # of 8 pieces, so a pair meets ceil(32 / 8) + 1 runs
    assert ns(32, 32, 8, 128, 4, 1020) == 5
    assert ns(1, 8, 1, 128, 0, 32) == 1           # one piece per pair
