"""The C ABI from plain C: tests/c/abi_host.c is compiled with gcc against
include/sinkattn.h, linked with libsinkattn.so and run (host-only entry
points; no device is touched)."""
import os
import shutil
import subprocess

import pytest

from learnable_sink_b200 import sinkattn as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_plain_c_program_uses_the_abi(tmp_path):
    if not os.path.exists(S.LIB_PATH):
        import learnable_sink_b200.build as B
        B.build()
    libdir = os.path.dirname(S.LIB_PATH)
    exe = str(tmp_path / "abi_host")
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Werror",
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c", "abi_host.c"),
                           "-L", libdir, "-lsinkattn", "-Wl,-rpath," + libdir, "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout
    kv = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert int(kv["version"]) >= 100
    assert kv["ok"] == '"ok"'
    assert int(kv["plan_bytes"]) > 0 and int(kv["plan_bytes_bad_heads"]) == 0
    assert int(kv["bwd_ws"]) > 0
    assert int(kv["decode_ws"]) >= 32 * 32 * 4 * 130 * 4
    assert int(kv["imp_ws"]) == 4 * 32 * 8
    assert int(kv["fwd_bad_d"]) == 1 and int(kv["gate_bad_t"]) == 1


def test_decode_schedule_keeps_partials_inside_the_workspace(tmp_path):
    """The streaming decode's static schedule (host code, compiled and run on
    the CPU): over many shapes, warp runs stay within the launched warps and
    no (sequence, KV head) pair meets more runs than its partial slots."""
    from learnable_sink_b200 import build as B
    exe = str(tmp_path / "decode_schedule_check")
    subprocess.check_call([B.nvcc(), "-std=c++17", "-arch=sm_100a", "-I",
                           os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c", "decode_schedule_check.cu"), "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout
    assert out.stdout.startswith("ok ")


def test_mask_span_and_sink_only_tile_match_elementwise_visibility(tmp_path):
    """The kernels' per-row mask (an interval plus the sink prefix) and the
    band's sink-only tile rule agree with the element-wise visibility
    predicate (host code, compiled and run on the CPU)."""
    from learnable_sink_b200 import build as B
    exe = str(tmp_path / "mask_span_check")
    subprocess.check_call([B.nvcc(), "-std=c++17", "-arch=sm_100a",
                           os.path.join(ROOT, "tests", "c", "mask_span_check.cu"), "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout
    assert out.stdout.startswith("ok ")
