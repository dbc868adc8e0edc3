#!/usr/bin/env python
"""Benchmark of the learnable-sink attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass over every hot-path stage on synthetic inputs:
  * training prefill (B=4 x T=4096 packed, Hq=32, Hkv=8, D=128, bf16, causal):
    tile schedule from the mask, forward (O, LSE_new, sink_s), backward
    (Delta/dsink preprocess, dK/dV/dQ kernel, dQ conversion) -- and, with N > 1
    ranks, the all-reduce of dsink (the sink is a parameter shared by every
    rank's queries);
  * StreamingLLM decode (32 sequences x 1 query, ring cache of 4 sink + 1020
    window slots, Hq=32, Hkv=8, D=128, bf16), after an L2 flush (write then
    read a buffer larger than L2, so no dirty lines are left to write back).
The headline value is the prefill fwd+bwd algorithmic throughput (visible
(query, key, head) triples x (4 + 10) x D flop) over all ranks; decode GB/s is
reported beside it.  Each rank processes its own batch (weak scaling).  Times
are CUDA events on the launching stream, max over ranks.

``--impl reference`` times the float64 CPU oracle (the correctness reference of
this repository) on the host cores on a bounded slice of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from learnable_sink_b200 import workloads as W  # noqa: E402

METRIC = "sink-attn fwd+bwd TFLOP/s & decode KV GB/s on 1 B200, % of roofline"
L2_BYTES = 126 * 1024 * 1024
# a device-side wait (about 0.5 ms at 1.9 GHz) enqueued before a short timed
# call, long enough for the host to issue that call behind it
HOST_COVER_CYCLES = 1_000_000
# launches of this library per step: plan 12, forward 1, backward 6
# (preprocess, dsink reduce, split-tile zero/finish, tensor-core kernel, dQ
# convert), decode 2
GPU_LAUNCHES_PER_STEP = 12 + 1 + 6 + 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def file_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def load_traffic(kernel, workload):
    """ncu-measured DRAM bytes per launch (profiles/traffic.json, keyed
    "kernel/workload"), valid only while the kernel's source is unchanged
    since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f).get(f"{kernel}/{workload}")
    if not t:
        return None
    src = os.path.join(ROOT, t["source"])
    if not os.path.exists(src) or file_hash(src) != t["source_sha256_16"]:
        return None
    return float(t["dram_bytes_per_launch"])


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of one GPU
    every 10 ms while running, through read-only NVML queries (nvidia-smi
    polling as a fallback).  Settings are only read, never changed."""

    # NVML clock-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index, period_s=0.01):
        self.index, self.period = device_index, period_s
        self.sm, self.mx, self.reasons = [], None, set()
        self.proc = self.thread = None
        self.stop = threading.Event()
        self.source = None

    def _pci_bus_id(self) -> bytes:
        """NVML's PCI bus id string ("domain:bus:device.0") of the CUDA device,
        built from the integer fields torch reports (CUDA and NVML may number
        devices differently)."""
        pr = torch.cuda.get_device_properties(self.index)
        dom, bus, dev = (int(pr.pci_domain_id), int(pr.pci_bus_id), int(pr.pci_device_id))
        return f"{dom:08X}:{bus:02X}:{dev:02X}.0".encode()

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        # the lookup takes a C string: pass bytes only (pynvml hands its
        # argument to c_char_p, which treats an integer as an address)
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(self._pci_bus_id())

    def _nvml_loop(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                bits = int(get_reasons(h))
                for b, n in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(n)
            except Exception:
                pass
            self.stop.wait(self.period)

    def _smi_read(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.proc.stdout:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                self.sm.append(float(parts[0]))
                self.mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    self.reasons.add(n)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.source = "nvml"
        except Exception:
            try:
                try:
                    which = self._pci_bus_id().decode()
                except Exception:
                    which = str(self.index)
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", which, f"--query-gpu={self.SMI_FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.thread = threading.Thread(target=self._smi_read, daemon=True)
                self.source = "nvidia-smi"
            except OSError:
                return self
        self.thread.start()
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self):
        sm = sorted(self.sm)
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": self.mx,
                "sm_min_mhz": sm[0] if sm else None, "reasons": sorted(self.reasons),
                "samples": len(sm), "source": self.source}


def init_dist(backend="nccl"):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                             **kw)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(inp, n_tok, n_groups):
    """Time the float64 oracle on sequence 0's first n_tok tokens and the
    first n_groups KV heads (with their query heads).  Returns (seconds,
    flop, description)."""
    import numpy as np
    import oracle
    T, Hq, Hkv, D = inp.shape
    G = Hq // Hkv
    sl = slice(0, n_tok)
    hq = slice(0, G * n_groups)
    hk = slice(0, n_groups)
    q, k, v = inp.q[sl, hq], inp.k[sl, hk], inp.v[sl, hk]
    do, a = inp.dout[sl, hq], inp.sink[hq]
    cu = np.array([0, n_tok], dtype=np.int32)
    t0 = time.perf_counter()
    oracle.fwd(q, k, v, a, inp.scale, causal=True, cu_seqlens=cu)
    oracle.bwd(q, k, v, a, do, inp.scale, causal=True, cu_seqlens=cu)
    dt = time.perf_counter() - t0
    pairs = n_tok * (n_tok + 1) // 2 * G * n_groups
    desc = (f"oracle fwd+bwd on sequence 0 tokens [0,{n_tok}) x {n_groups} KV head(s) "
            f"({G * n_groups} query heads) of the prefill workload, float64, "
            f"{oracle.num_threads()} OpenMP threads")
    return dt, pairs * 14 * D, desc, oracle.num_threads()


def run_reference(args, world, rank):
    base = {"metric": METRIC, "unit": "TFLOP/s", "higher_is_better": True, "impl": "reference"}
    if rank != 0:
        return
    inp = W.prefill()
    n_tok, n_groups = 2048, 1
    for _ in range(args.warmup):
        cpu_oracle_sample(inp, n_tok, n_groups)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl, desc, cores = cpu_oracle_sample(inp, n_tok, n_groups)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = dict(base, value=value, n_gpus=world, steps=args.steps, warmup=args.warmup,
                ms_per_step=tot_t / args.steps * 1e3, scaling="weak", vs_baseline=None,
                dtype="f64", data="synthetic",
                config={"workload": "training prefill B4 T4096 Hq32 Hkv8 D128 causal fwd+bwd",
                        "sample": desc},
                cpu_baseline={"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                              "sample": desc},
                e2e={"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                     "d2h_bytes_per_step": 0})
    print(json.dumps(line), flush=True)


def executed_pairs(plan, Hq, Hkv):
    """(query, key, head) triples of the tiles the plan lists (visible or
    masked inside a partial tile): the work the kernels execute, read from the
    plan header's entry count (int32 word 12) and tile size (word 4); a list
    entry covers tile x tile pairs for every query head of its KV-head slot."""
    h = plan.buf[:64].cpu().view(torch.int32).tolist()
    tile, kh_slots, n_entries = h[4], h[5], h[12]
    heads = Hq if kh_slots == 1 else Hq // Hkv
    return n_entries * tile * tile * heads


def measure_config(S, inp, dev, steps=10, warmup=3):
    """Plan+fwd+bwd of one workload: per-call and per-kernel times (CUDA events)."""
    T, Hq, Hkv, D = inp.shape
    pairs = W.visible_pairs(inp.mask, Hq, Hkv)
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    sink, dout = inp.sink.to(dev), inp.dout.to(dev)
    mask = S.Mask.from_spec(inp.mask, dev)
    plan = S.Plan(T, Hq, Hkv, mask)
    out = torch.empty_like(q)
    lse = torch.empty(T, Hq, dtype=torch.float32, device=dev)
    ss = torch.empty_like(lse)
    ws = torch.empty(S.bwd_workspace_bytes(q, k, mask), dtype=torch.uint8, device=dev)

    def step():
        plan.rebuild()
        S.fwd(q, k, v, sink, mask, plan, scale=inp.scale, out=out, lse=lse, sink_s=ss)
        S.bwd(q, k, v, out, dout, lse, sink, mask, plan, scale=inp.scale, workspace=ws)

    for _ in range(warmup):
        step()
    ev = {n: [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
          for n in ("s0", "s1", "f0", "f1", "b0", "b1")}
    for lst in ev.values():
        for e in lst:
            e.record()
    torch.cuda.synchronize()
    for i in range(steps):
        S.set_kernel_events(S.KERNEL_FWD, ev["f0"][i], ev["f1"][i])
        S.set_kernel_events(S.KERNEL_BWD, ev["b0"][i], ev["b1"][i])
        ev["s0"][i].record()
        step()
        ev["s1"][i].record()
    torch.cuda.synchronize()
    S.set_kernel_events(S.KERNEL_FWD, None, None)
    S.set_kernel_events(S.KERNEL_BWD, None, None)

    def mean(a, b):
        return sum(x.elapsed_time(y) for x, y in zip(ev[a], ev[b])) / steps

    step_ms, f_ms, b_ms = mean("s0", "s1"), mean("f0", "f1"), mean("b0", "b1")
    ex = executed_pairs(plan, Hq, Hkv)
    return {"workload": inp.name, "visible_pairs": pairs, "D": D, "executed_pairs": ex,
            "executed_fwd_tflops": 4 * D * ex / (f_ms * 1e-3) / 1e12,
            "executed_bwd_tflops": 10 * D * ex / (b_ms * 1e-3) / 1e12,
            "plan_fwd_bwd_ms": step_ms, "tflops": 14 * D * pairs / (step_ms * 1e-3) / 1e12,
            "fwd_kernel_ms": f_ms, "fwd_kernel_tflops": 4 * D * pairs / (f_ms * 1e-3) / 1e12,
            "bwd_kernel_ms": b_ms, "bwd_kernel_tflops": 10 * D * pairs / (b_ms * 1e-3) / 1e12}


def measure_decode_kernel(S, decode_step, flush, flush_rd, reps=20):
    """Median CUDA-event time of the decode's streaming kernel, L2 flushed
    before each call."""
    ts = []
    for _ in range(reps):
        flush.zero_()
        flush_rd.sum()
        torch.cuda._sleep(HOST_COVER_CYCLES)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        e1.record()
        S.set_kernel_events(S.KERNEL_DECODE, e0, e1)
        decode_step()
        S.set_kernel_events(S.KERNEL_DECODE, None, None)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return sorted(ts)[len(ts) // 2]


def measure_fp8_decode(S, dec, dev, flush, flush_rd, reps=20):
    """The FP8 window-cache decode on the StreamingLLM decode workload (the
    same cache with its window slots as E4M3 codes): median CUDA-event time
    of the whole call and of its streaming kernel, L2 flushed before each
    call, and the call's algorithmic bytes (filled sink rows in bf16, filled
    window rows as codes, Q/O bf16, LSE and sink_s)."""
    cache = [t.to(dev) for t in W.fp8_window_cache(dec, seed=W.SEED_BASE + 501)]
    q, cs, sink = dec.q.to(dev), dec.cache_seqlens.to(dev), dec.sink.to(dev)
    B, Hq, D = dec.q.shape
    Hkv = dec.k_cache.shape[2]
    n = torch.clamp(dec.cache_seqlens.long(), min=0, max=dec.n_sink + dec.window)
    sink_rows = int(torch.clamp(n, max=dec.n_sink).sum())
    win_rows = int((n - torch.clamp(n, max=dec.n_sink)).sum())
    kv_bytes = 2 * Hkv * D * (2 * sink_rows + win_rows)
    nbytes = kv_bytes + 2 * B * Hq * D * 2 + 2 * B * Hq * 4 + B * 4 + 2 * Hkv * 4
    splits = S.decode_fp8_num_splits(B, Hq, Hkv, D, dec.n_sink, dec.window)
    ws = torch.empty(S.decode_workspace_bytes(B, Hq, D, splits), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    ss = torch.empty_like(lse)

    def call():
        S.decode_fp8(q, *cache, cs, dec.n_sink, dec.window, sink, scale=dec.scale,
                     num_splits=splits, workspace=ws, out=out, lse=lse, sink_s=ss)

    for _ in range(3):
        call()
    res = {}
    for mode in ("call", "kernel"):
        ts = []
        for _ in range(reps):
            flush.zero_()
            flush_rd.sum()
            torch.cuda._sleep(HOST_COVER_CYCLES)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            if mode == "kernel":
                e1.record()
                S.set_kernel_events(S.KERNEL_DECODE, e0, e1)
            call()
            if mode == "kernel":
                S.set_kernel_events(S.KERNEL_DECODE, None, None)
            else:
                e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        res[mode + "_ms"] = sorted(ts)[len(ts) // 2]
    res.update(bytes=nbytes, kernel_bytes=kv_bytes, num_splits=splits,
               call_gbs=nbytes / (res["call_ms"] * 1e-3) / 1e9)
    return res


def measure_gates(S, q, k, lse, sink_s, mask, scale, flush, flush_rd, hbm_gbs, reps=10):
    """Gate rows on the prefill's tensors: the sink-free model's gate (reads Q
    once) and the head importance (reads sink_s once).  L2 is flushed before
    each call, then the device is kept busy (torch.cuda._sleep) while the host
    issues the call, so the CUDA events around it see no host issue gap."""
    T, Hq, D = q.shape
    gate = torch.empty(T, Hq, dtype=torch.float32, device=q.device)
    imp = torch.empty(Hq, dtype=torch.float32, device=q.device)
    iws = torch.empty(max(16, S.lib().sinkattn_gate_importance_workspace_bytes(T, Hq)),
                      dtype=torch.uint8, device=q.device)
    n_seq = mask.cu_seqlens.numel() - 1
    res = {}
    for name, call, nbytes in (
            ("gate_vanilla", lambda: S.gate_vanilla(q, k, lse, mask, scale=scale, gate=gate),
             q.numel() * q.element_size() + 8 * T * Hq + n_seq * k.shape[1] * D * k.element_size()),
            ("gate_importance", lambda: S.gate_importance(sink_s, workspace=iws, imp=imp),
             4 * T * Hq)):
        for _ in range(3):
            call()
        ts = []
        for _ in range(reps):
            flush.zero_()
            flush_rd.sum()
            torch.cuda._sleep(HOST_COVER_CYCLES)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = sorted(ts)[len(ts) // 2]
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"ms": ms, "bytes": nbytes, "achieved_gbs": gbs, "frac_of_hbm": gbs / hbm_gbs}
    return res


def run_profile_workload(args, dev):
    """Launches of one workload's kernels for an external profiler (warm-up +
    steps, nothing timed, no JSON line): the band or varlen block-sparse
    plan+fwd+bwd, or the FP8 window-cache decode."""
    from learnable_sink_b200 import sinkattn as S
    torch.cuda.set_device(dev)
    if args.profile_workload in ("band", "varlen"):
        inp = W.band() if args.profile_workload == "band" else W.varlen()
        T, Hq, Hkv, D = inp.shape
        q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
        sink, dout = inp.sink.to(dev), inp.dout.to(dev)
        mask = S.Mask.from_spec(inp.mask, dev)
        plan = S.Plan(T, Hq, Hkv, mask)
        out = torch.empty_like(q)
        lse = torch.empty(T, Hq, dtype=torch.float32, device=dev)
        ss = torch.empty_like(lse)
        ws = torch.empty(S.bwd_workspace_bytes(q, k, mask), dtype=torch.uint8, device=dev)

        def step():
            plan.rebuild()
            S.fwd(q, k, v, sink, mask, plan, scale=inp.scale, out=out, lse=lse, sink_s=ss)
            S.bwd(q, k, v, out, dout, lse, sink, mask, plan, scale=inp.scale, workspace=ws)
    elif args.profile_workload == "gate":
        inp = W.prefill()
        T, Hq, Hkv, D = inp.shape
        q, k = inp.q.to(dev), inp.k.to(dev)
        mask = S.Mask.from_spec(inp.mask, dev)
        lse = torch.randn(T, Hq, dtype=torch.float32, device=dev).abs_().add_(4.0)
        gate = torch.empty(T, Hq, dtype=torch.float32, device=dev)

        def step():
            S.gate_vanilla(q, k, lse, mask, scale=inp.scale, gate=gate)
    else:  # fp8 decode
        dec = W.decode()
        cache = [t.to(dev) for t in W.fp8_window_cache(dec, seed=W.SEED_BASE + 501)]
        qd, cs, dsk = dec.q.to(dev), dec.cache_seqlens.to(dev), dec.sink.to(dev)

        def step():
            S.decode_fp8(qd, *cache, cs, dec.n_sink, dec.window, dsk, scale=dec.scale)
    for _ in range(args.warmup + args.steps):
        step()
    torch.cuda.synchronize()


def run_ours(args, world, rank, local):
    from learnable_sink_b200 import sinkattn as S
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.profile_workload:
        return run_profile_workload(args, dev)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()

    # ---- prefill inputs (per rank: its own batch)
    inp = W.prefill(seed_offset=1000 * rank)
    T, Hq, Hkv, D = inp.shape
    pairs = W.visible_pairs(inp.mask, Hq, Hkv)
    flop_fwd, flop_bwd = 4 * D * pairs, 10 * D * pairs
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    sink, dout = inp.sink.to(dev), inp.dout.to(dev)
    mask = S.Mask.from_spec(inp.mask, dev)
    plan = S.Plan(T, Hq, Hkv, mask)
    out = torch.empty_like(q)
    lse = torch.empty(T, Hq, dtype=torch.float32, device=dev)
    sink_s = torch.empty_like(lse)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dsink = torch.empty(Hq, dtype=torch.float32, device=dev)
    ws = torch.empty(S.bwd_workspace_bytes(q, k, mask), dtype=torch.uint8, device=dev)

    # ---- decode inputs
    dec = W.decode(seed_offset=1000 * rank)
    dq_in = dec.q.to(dev)
    kc, vc = dec.k_cache.to(dev), dec.v_cache.to(dev)
    cs, dsk = dec.cache_seqlens.to(dev), dec.sink.to(dev)
    B, dHq, dD = dec.q.shape
    dHkv = dec.k_cache.shape[2]
    n_splits = S.decode_num_splits(B, dHq, dHkv, dD, dec.n_sink, dec.window)
    dws = torch.empty(S.decode_workspace_bytes(B, dHq, dD, n_splits), dtype=torch.uint8, device=dev)
    dout_dec = torch.empty_like(dq_in)
    dlse = torch.empty(B, dHq, dtype=torch.float32, device=dev)
    dss = torch.empty_like(dlse)
    valid = torch.clamp(dec.cache_seqlens, max=dec.n_sink + dec.window).sum().item()
    dec_bytes = 2 * valid * dHkv * dD * 2 + 2 * B * dHq * dD * 2 + 2 * B * dHq * 4 + B * 4
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def prefill_step(bufs=None):
        qq, kk, vv, dd, ss = ((q, k, v, dout, sink) if bufs is None else
                              (bufs["q"], bufs["k"], bufs["v"], bufs["dout"], bufs["sink"]))
        plan.rebuild()
        S.fwd(qq, kk, vv, ss, mask, plan, scale=inp.scale, out=out, lse=lse, sink_s=sink_s)
        S.bwd(qq, kk, vv, out, dd, lse, ss, mask, plan, scale=inp.scale, workspace=ws,
              dq=dq, dk=dk, dv=dv, dsink=dsink)
        if world > 1:
            torch.distributed.all_reduce(dsink)

    def decode_step():
        S.decode(dq_in, kc, vc, cs, dec.n_sink, dec.window, dsk, scale=dec.scale,
                 num_splits=n_splits, workspace=dws, out=dout_dec, lse=dlse, sink_s=dss)

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        return e

    # warm-up (also creates every event handle)
    for _ in range(args.warmup):
        prefill_step()
        flush.zero_()
        decode_step()
    torch.cuda.synchronize()
    if args.profile:  # launches for an external profiler only; nothing is timed
        for _ in range(args.steps):
            prefill_step()
            decode_step()
        torch.cuda.synchronize()
        return

    K = args.steps
    evs = {n: [ev() for _ in range(K)] for n in
           ("p0", "p1", "d0", "d1", "kf0", "kf1", "kb0", "kb1")}
    host_t = [0.0, 0.0]
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        host_t[0] = time.perf_counter()
        r0 = ev()
        for i in range(K):
            S.set_kernel_events(S.KERNEL_FWD, evs["kf0"][i], evs["kf1"][i])
            S.set_kernel_events(S.KERNEL_BWD, evs["kb0"][i], evs["kb1"][i])
            evs["p0"][i].record()
            prefill_step()
            evs["p1"][i].record()
            # decode's working set is about L2-sized: start it cold.  Writing a
            # buffer larger than L2 evicts it; reading a second one then writes
            # those dirty lines back before the decode starts, so their
            # write-back traffic is not charged to the decode.
            flush.zero_()
            flush_rd.sum()
            evs["d0"][i].record()
            decode_step()
            evs["d1"][i].record()
        r1 = ev()
        host_t[1] = time.perf_counter()
        torch.cuda.synchronize()
    for w in (S.KERNEL_FWD, S.KERNEL_BWD):
        S.set_kernel_events(w, None, None)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    code = S.get_status()
    if code != 0:
        raise RuntimeError(f"device status {S.ERR_NAMES.get(code, code)}")

    def total(a, b):
        return sum(x.elapsed_time(y) for x, y in zip(evs[a], evs[b]))

    region_ms = max_over_ranks(r0.elapsed_time(r1), world)
    prefill_ms = max_over_ranks(total("p0", "p1"), world)
    decode_ms = max_over_ranks(total("d0", "d1"), world)
    # the rest of the step: the L2 flush between prefill and decode, and the
    # device's idle time from one step's decode to the next step's prefill
    flush_only_ms = total("p1", "d0") / K
    between_ms = sum(evs["d1"][i].elapsed_time(evs["p0"][i + 1]) for i in range(K - 1)) / max(1, K - 1)
    kf_ms = total("kf0", "kf1") / K
    kb_ms = total("kb0", "kb1") / K
    # the streaming kernel alone (its own events; the step loop above times
    # whole decode calls without events between their launches)
    kd_ms = measure_decode_kernel(S, decode_step, flush, flush_rd)
    value = world * K * (flop_fwd + flop_bwd) / (prefill_ms * 1e-3) / 1e12
    dec_gbs = world * K * dec_bytes / (decode_ms * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers
    pin = {n: t.cpu().pin_memory() for n, t in (("q", inp.q), ("k", inp.k), ("v", inp.v),
                                                 ("dout", inp.dout), ("sink", inp.sink))}
    h_dsink = torch.empty(Hq, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = h_dsink.numel() * 4

    # Double-buffered inputs: the host-to-device copies of step i + 1 run on a
    # second stream while step i computes; every step's inputs are still
    # copied inside the timed region, and dsink is read back after each step.
    bufs = [dict(q=q, k=k, v=v, dout=dout, sink=sink),
            {n: torch.empty_like(t) for n, t in (("q", q), ("k", k), ("v", v),
                                                 ("dout", dout), ("sink", sink))}]
    copy_stream = torch.cuda.Stream(device=dev)
    landed = [torch.cuda.Event() for _ in range(2)]
    released = [torch.cuda.Event() for _ in range(2)]

    def issue_copies(b):
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(released[b])
            for n in ("q", "k", "v", "dout", "sink"):
                bufs[b][n].copy_(pin[n], non_blocking=True)
            landed[b].record(copy_stream)

    def compute(b):
        stream.wait_event(landed[b])
        prefill_step(bufs[b])
        released[b].record(stream)
        h_dsink.copy_(dsink, non_blocking=True)

    def e2e_run(n):
        e0 = ev()
        copy_stream.wait_event(e0)
        issue_copies(0)
        for j in range(n):
            if j + 1 < n:
                issue_copies((j + 1) % 2)
            compute(j % 2)
        return e0, ev()

    for e in released:
        e.record(stream)
    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    K2 = max(3, K // 2)
    e0, e1 = e2e_run(K2)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = world * K2 * (flop_fwd + flop_bwd) / (e2e_ms * 1e-3) / 1e12

    if rank != 0:
        return
    gates = measure_gates(S, q, k, lse, sink_s, mask, inp.scale, flush, flush_rd,
                          peaks["hbm_gbs"])
    clocks = clk.summary()
    burst, sustained, hbm = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"], peaks["hbm_gbs"]
    # The timed region lasts well under the seconds-long loop the sustained
    # figure was taken over; the clock sampled during it says which applies.
    at_max = (clocks["sm_mhz"] is not None and clocks["sm_max_mhz"] is not None
              and clocks["sm_mhz"] >= 0.95 * clocks["sm_max_mhz"])
    region_s = region_ms * 1e-3
    tensor_peak = burst if (at_max or region_s < 2.0) else sustained
    tensor_peak_name = "bf16_tflops (burst)" if tensor_peak == burst else "bf16_tflops_sustained"
    dec_kernel_bytes = 2 * valid * dHkv * dD * 2

    def tensor_entry(kernel, workload, ms, flop):
        ach = flop / (ms * 1e-3) / 1e12
        return {"kernel": kernel, "workload": workload, "bound": "tensor", "achieved": ach,
                "peak": tensor_peak, "unit": "TFLOP/s", "frac": ach / tensor_peak,
                "frac_of_sustained": ach / sustained, "ms": ms,
                "traffic": load_traffic(kernel, workload)}

    def hbm_entry(kernel, workload, ms, nbytes):
        ach = nbytes / (ms * 1e-3) / 1e9
        return {"kernel": kernel, "workload": workload, "bound": "hbm", "achieved": ach,
                "peak": hbm, "unit": "GB/s", "frac": ach / hbm, "frac_of_8tbs": ach / 8000.0,
                "ms": ms, "bytes": nbytes, "traffic": load_traffic(kernel, workload)}

    fp8 = measure_fp8_decode(S, dec, dev, flush, flush_rd)
    rooflines = [
        tensor_entry("fwd_tc_kernel", "training_prefill", kf_ms, flop_fwd),
        tensor_entry("bwd_tc_kernel", "training_prefill", kb_ms, flop_bwd),
        hbm_entry("decode_warp_kernel", "streamingllm_decode", kd_ms, dec_kernel_bytes),
        hbm_entry("decode call (stream + merge)", "streamingllm_decode", decode_ms / K, dec_bytes),
        hbm_entry("decode_fp8_kernel", "streamingllm_decode_fp8_window", fp8["kernel_ms"],
                  fp8["kernel_bytes"]),
        hbm_entry("decode_fp8 call (stream + merge)", "streamingllm_decode_fp8_window",
                  fp8["call_ms"], fp8["bytes"]),
        hbm_entry("gate_vanilla_kernel", "training_prefill", gates["gate_vanilla"]["ms"],
                  gates["gate_vanilla"]["bytes"]),
    ]
    extra = []
    if args.configs:
        for mk, wl in ((W.band, "streamingllm_band"), (W.varlen, "varlen_block_sparse")):
            r = measure_config(S, mk(), dev)
            r["frac"] = r["tflops"] / tensor_peak
            extra.append(r)
            D_ = r["D"]
            rooflines.append(tensor_entry("fwd_tc_kernel", wl, r["fwd_kernel_ms"],
                                          4 * D_ * r["visible_pairs"]))
            rooflines.append(tensor_entry("bwd_tc_kernel", wl, r["bwd_kernel_ms"],
                                          10 * D_ * r["visible_pairs"]))
    dominant = rooflines[1]  # bwd_tc_kernel: the largest share of the prefill step
    flush_ms = region_ms / K - prefill_ms / K - decode_ms / K
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": region_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": "training prefill B4 T4096 Hq32 Hkv8 D128 bf16 causal, plan+fwd+bwd "
                        "(+ StreamingLLM decode B32 cache 4+1020 Hq32 Hkv8 D128 per step)",
            "global_batch": 4 * world, "seq_len": 4096, "parallelism": f"dp{world}",
            "visible_pairs_per_rank": pairs,
            "executed_pairs_per_rank": executed_pairs(plan, Hq, Hkv),
            "l2": "prefill inputs larger than L2; before each decode L2 is flushed by writing "
                  "252 MB and then reading another 252 MB (dirty lines written back before "
                  "the decode starts)",
        },
        "decode": {"value": dec_gbs, "unit": "GB/s", "ms_per_call": decode_ms / K,
                   "bytes_per_call": dec_bytes, "num_splits": n_splits,
                   "frac": dec_gbs / hbm, "frac_of_8tbs": dec_gbs / 8000.0},
        "decode_fp8_window": fp8,
        "step_breakdown_ms": {
            "prefill": prefill_ms / K, "decode_call": decode_ms / K,
            "l2_flush_and_gaps": flush_ms, "l2_flush": flush_only_ms,
            "decode_to_next_prefill": between_ms,
            "host_issue_per_step": (host_t[1] - host_t[0]) * 1e3 / K,
            "note": "device time per step; l2_flush_and_gaps = step - prefill - decode "
                    "(the two flush kernels between prefill and decode, and any idle time); "
                    "l2_flush = prefill end to decode start; decode_to_next_prefill = decode "
                    "end to the next step's prefill start"},
        "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": K2,
                "what": "pinned-host q,k,v,dO,sink -> device (step i+1's copies on a second stream "
                        "overlap step i's compute, double-buffered), plan+fwd+bwd, dsink -> host"},
        "gpu_launches": K * GPU_LAUNCHES_PER_STEP,
        "roofline": dict(dominant, peak_source=f"{peak_src} {tensor_peak_name}",
                         algorithmic="10*D flop per visible (query, key, head) triple x visible "
                                     "triples per launch"),
        "rooflines": rooflines,
        # gate rows, timed after the main region on the prefill's tensors
        # (median of 10 calls): not part of the step
        "gates": gates,
    }
    if extra:
        line["other_configs"] = extra
    if world == 1:
        dt, fl, desc, cores = cpu_oracle_sample(inp, 4096, 2)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": cores,
                                "kind": "oracle", "sample": desc, "seconds": dt}
    print(json.dumps(line), flush=True)


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(n: int, argv, skip_device_check: bool) -> int:
    """``--gpus N`` without a launcher: start N processes of this script, one
    per GPU, with the environment torch.distributed.run would give them
    (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR/PORT on 127.0.0.1).  Only rank 0
    prints.  Returns the first non-zero exit code of a rank, else 0."""
    if not skip_device_check:
        have = torch.cuda.device_count()
        if n > have:
            print(f"bench.py: --gpus {n} but only {have} CUDA device(s) are visible",
                  file=sys.stderr)
            return 2
    port = free_port()
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n),
                   LOCAL_WORLD_SIZE=str(n), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, os.path.abspath(__file__)] + list(argv),
                                      env=env))
    rc = 0
    try:
        for p in procs:
            code = p.wait()
            if code != 0 and rc == 0:
                rc = code
                for q in procs:  # a failed rank: stop the others (exact children only)
                    if q.poll() is None:
                        q.terminate()
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
                p.wait()
    return rc


def run_dry(args, world, rank):
    """Launcher check without CUDA: every rank joins a gloo group, all-reduces
    its rank number and meets a barrier; rank 0 prints one line."""
    t = torch.tensor([float(rank + 1)])
    torch.distributed.all_reduce(t)
    torch.distributed.barrier()
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_gpus": world, "rank_sum": float(t.item()),
                          "master_addr": os.environ.get("MASTER_ADDR"),
                          "local_rank": int(os.environ.get("LOCAL_RANK", "0"))}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--profile", action="store_true",
                    help="run warm-up + steps of the prefill and decode stages for a profiler "
                         "(no timing, no JSON line)")
    ap.add_argument("--profile-workload", choices=["band", "varlen", "fp8", "gate"], default=None,
                    help="like --profile, for one other workload's kernels")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the band / varlen block-sparse measurements")
    ap.add_argument("--dry-run", action="store_true",
                    help="launcher check on CPU: gloo ranks, no CUDA calls")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # the reference arm runs on the host cores: no GPU count to check
        sys.exit(launch_ranks(args.gpus, sys.argv[1:], args.dry_run or args.impl == "reference"))
    if args.dry_run:
        world, rank, _ = init_dist(backend="gloo")
        try:
            run_dry(args, world, rank)
        finally:
            if world > 1:
                torch.distributed.destroy_process_group()
        return
    world, rank, local = init_dist() if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
