"""Learnable-sink GQA attention for B200 (sm_100a).

The compute lives in ``libsinkattn.so`` (hand-written CUDA behind a C ABI,
declared in ``include/sinkattn.h``); :mod:`learnable_sink_b200.sinkattn` is the
thin ctypes binding.  :mod:`learnable_sink_b200.workloads` draws the seeded
synthetic inputs.
"""
__all__ = ["sinkattn", "workloads"]
