"""Seeded synthetic inputs for learnable-sink attention.

This module only draws random inputs and shapes them; it holds none of the
attention arithmetic.  Both the CUDA path and the float64 oracle take their
inputs from here, so the two see bit-identical rounded values.

Workloads (all synthetic; no dataset is involved):

* ``tiny``     B=1, T=128, Hq=4, Hkv=2, D=64, fp32, causal.
* ``decode``   32 sequences x 1 query, ring cache of 4 sink slots + 1020
               window slots (StreamingLLM's four initial tokens), Hq=32,
               Hkv=8, D=128, bf16; tokens ever appended ~ U[1024, 1e6], so the
               ring head sits at a random offset in every sequence.
* ``prefill``  B=4 x T=4096 (uniform packed sequences), Hq=32, Hkv=8, D=128,
               bf16, causal, sink ~ N(0, 0.5).
* ``band``     T=16384, Hq=32, Hkv=8, D=128, bf16, causal, n_sink=4,
               window=2048 (keys 0..3 plus the last 2048 causal positions).
* ``varlen``   T_tot=32768 packed from lengths ~ U[512, 8192] (the last
               length truncated so the total is exact), Hq=64, Hkv=8, D=64,
               bf16; per (sequence-local 64-query block, KV head): 16 distinct
               random earlier 64-key blocks (all of them if fewer) plus the
               diagonal block.

Q/K/V/dO ~ N(0, 1) drawn in fp32 on a CPU ``torch.Generator`` and rounded
to the run dtype; the learnable sink ~ N(0, sigma) in fp32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

SEED_BASE = 20261202


@dataclasses.dataclass
class MaskSpec:
    causal: bool = True
    n_sink: int = 0
    window: int = 0
    cu_seqlens: Optional[torch.Tensor] = None  # int32 [n_seq+1] (CPU)
    block_indices: Optional[torch.Tensor] = None  # int32 [Hkv, n_qblk, max_blocks]
    block_q: int = 64
    block_k: int = 64

    @property
    def n_seq(self) -> int:
        return int(self.cu_seqlens.numel()) - 1

    @property
    def max_seqlen(self) -> int:
        return int((self.cu_seqlens[1:] - self.cu_seqlens[:-1]).max())

    def oracle_kwargs(self) -> dict:
        """The mask as the oracle's keyword arguments (numpy int32)."""
        return dict(causal=self.causal, n_sink=self.n_sink, window=self.window,
                    cu_seqlens=self.cu_seqlens.numpy(),
                    block_indices=None if self.block_indices is None
                    else self.block_indices.numpy(),
                    block_q=self.block_q, block_k=self.block_k)


@dataclasses.dataclass
class AttnInputs:
    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    sink: Optional[torch.Tensor]
    dout: Optional[torch.Tensor]
    mask: MaskSpec
    scale: float

    @property
    def shape(self):
        T, Hq, D = self.q.shape
        return T, Hq, self.k.shape[1], D


@dataclasses.dataclass
class DecodeInputs:
    name: str
    q: torch.Tensor          # [B, Hq, D]
    k_cache: torch.Tensor    # [B, S, Hkv, D]
    v_cache: torch.Tensor
    cache_seqlens: torch.Tensor  # int32 [B]
    n_sink: int
    window: int
    sink: Optional[torch.Tensor]
    scale: float


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _normal(gen, shape, dtype, std=1.0):
    return (torch.randn(*shape, generator=gen, dtype=torch.float32) * std).to(dtype)


def uniform_cu_seqlens(n_seq: int, seqlen: int) -> torch.Tensor:
    return torch.arange(0, (n_seq + 1) * seqlen, seqlen, dtype=torch.int32)


def random_cu_seqlens(total: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """Lengths ~ U[lo, hi] until the total is reached; the last length is
    truncated so the lengths sum to ``total`` exactly."""
    rng = np.random.default_rng(seed)
    lens, acc = [], 0
    while acc < total:
        n = int(rng.integers(lo, hi + 1))
        n = min(n, total - acc)
        lens.append(n)
        acc += n
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return torch.from_numpy(cu)


def random_block_indices(cu_seqlens: torch.Tensor, Hkv: int, block_q: int,
                         block_k: int, n_random: int, seed: int,
                         shuffle: bool = False) -> torch.Tensor:
    """Per (KV head, sequence-local query block): ``n_random`` distinct random
    earlier key blocks (all of them if fewer exist) plus the diagonal block,
    padded with -1 to ``n_random + 1`` entries.  Block ids are sequence-local.
    Requires block_q == block_k (the diagonal block is the query block)."""
    assert block_q == block_k
    rng = np.random.default_rng(seed)
    lens = (cu_seqlens[1:] - cu_seqlens[:-1]).tolist()
    nqb = [(l + block_q - 1) // block_q for l in lens]
    total = sum(nqb)
    mb = n_random + 1
    bi = np.full((Hkv, total, mb), -1, dtype=np.int32)
    for g in range(Hkv):
        r = 0
        for s, nb in enumerate(nqb):
            for qb in range(nb):
                if qb <= n_random:
                    chosen = np.arange(qb, dtype=np.int32)
                else:
                    chosen = np.sort(rng.choice(qb, size=n_random, replace=False)).astype(np.int32)
                row = np.concatenate([chosen, np.array([qb], dtype=np.int32)])
                if shuffle:
                    row = rng.permutation(row)
                bi[g, r, :len(row)] = row
                r += 1
    return torch.from_numpy(bi)


def make_attn(name: str, *, T_tot: int, Hq: int, Hkv: int, D: int, dtype,
              mask: MaskSpec, seed: int, sink_std: Optional[float] = 1.0,
              with_dout: bool = True, sink_values=None) -> AttnInputs:
    gen = _gen(seed)
    q = _normal(gen, (T_tot, Hq, D), dtype)
    k = _normal(gen, (T_tot, Hkv, D), dtype)
    v = _normal(gen, (T_tot, Hkv, D), dtype)
    if sink_values is not None:
        sink = torch.as_tensor(sink_values, dtype=torch.float32).reshape(Hq).clone()
    elif sink_std is None:
        sink = None
    else:
        sink = _normal(gen, (Hq,), torch.float32, sink_std)
    dout = _normal(gen, (T_tot, Hq, D), dtype) if with_dout else None
    return AttnInputs(name, q, k, v, sink, dout, mask, 1.0 / math.sqrt(D))


def tiny(seed_offset: int = 0) -> AttnInputs:
    return make_attn("tiny B1 T128 Hq4 Hkv2 D64 fp32 causal", T_tot=128, Hq=4,
                     Hkv=2, D=64, dtype=torch.float32,
                     mask=MaskSpec(causal=True, cu_seqlens=uniform_cu_seqlens(1, 128)),
                     seed=SEED_BASE + 0 + seed_offset)


def prefill(n_seq: int = 4, seqlen: int = 4096, seed_offset: int = 0) -> AttnInputs:
    return make_attn(f"training prefill B{n_seq} T{seqlen} Hq32 Hkv8 D128 bf16 causal",
                     T_tot=n_seq * seqlen, Hq=32, Hkv=8, D=128, dtype=torch.bfloat16,
                     mask=MaskSpec(causal=True, cu_seqlens=uniform_cu_seqlens(n_seq, seqlen)),
                     seed=SEED_BASE + 2 + seed_offset, sink_std=0.5)


def band(T: int = 16384, n_sink: int = 4, window: int = 2048,
         seed_offset: int = 0) -> AttnInputs:
    return make_attn(f"StreamingLLM band T{T} n_sink{n_sink} window{window} Hq32 Hkv8 D128 bf16",
                     T_tot=T, Hq=32, Hkv=8, D=128, dtype=torch.bfloat16,
                     mask=MaskSpec(causal=True, n_sink=n_sink, window=window,
                                   cu_seqlens=uniform_cu_seqlens(1, T)),
                     seed=SEED_BASE + 3 + seed_offset)


def varlen(T_tot: int = 32768, lo: int = 512, hi: int = 8192, Hq: int = 64,
           Hkv: int = 8, D: int = 64, n_random: int = 16,
           seed_offset: int = 0) -> AttnInputs:
    seed = SEED_BASE + 4 + seed_offset
    cu = random_cu_seqlens(T_tot, lo, hi, seed)
    bi = random_block_indices(cu, Hkv, 64, 64, n_random, seed + 1)
    return make_attn(f"packed varlen block-sparse T{T_tot} Hq{Hq} Hkv{Hkv} D{D} bf16",
                     T_tot=T_tot, Hq=Hq, Hkv=Hkv, D=D, dtype=torch.bfloat16,
                     mask=MaskSpec(causal=True, cu_seqlens=cu, block_indices=bi,
                                   block_q=64, block_k=64, n_sink=0, window=0),
                     seed=seed)


def decode(B: int = 32, n_sink: int = 4, window: int = 1020, Hq: int = 32,
           Hkv: int = 8, D: int = 128, dtype=torch.bfloat16,
           seqlen_range=(1024, 1_000_000), seed_offset: int = 0,
           sink_std: Optional[float] = 1.0) -> DecodeInputs:
    seed = SEED_BASE + 1 + seed_offset
    gen = _gen(seed)
    S = n_sink + window
    q = _normal(gen, (B, Hq, D), dtype)
    kc = _normal(gen, (B, S, Hkv, D), dtype)
    vc = _normal(gen, (B, S, Hkv, D), dtype)
    lo, hi = seqlen_range
    cs = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64).to(torch.int32)
    sink = None if sink_std is None else _normal(gen, (Hq,), torch.float32, sink_std)
    return DecodeInputs(f"StreamingLLM decode B{B} cache {n_sink}+{window} Hq{Hq} Hkv{Hkv} D{D}",
                        q, kc, vc, cs, n_sink, window, sink, 1.0 / math.sqrt(D))


def visible_pairs(spec: MaskSpec, Hq: int, Hkv: int) -> int:
    """Number of visible (query, key, query-head) triples of a mask: the unit
    of algorithmic work (forward 4*D flop each, backward 10*D).  Counted from
    closed forms per sequence (causal / StreamingLLM band) or per selected
    block; bookkeeping only."""
    lens = (spec.cu_seqlens[1:] - spec.cu_seqlens[:-1]).tolist()
    G = Hq // Hkv
    if spec.block_indices is None:
        total = 0
        for L in lens:
            i = np.arange(L, dtype=np.int64)
            if not spec.causal:
                total += L * L
            elif spec.window <= 0:
                total += L * (L + 1) // 2
            else:
                win = np.minimum(i + 1, spec.window)
                sink = np.minimum(spec.n_sink, np.maximum(0, i + 1 - spec.window))
                total += int((win + sink).sum())
        return int(total) * Hq
    bq, bk = spec.block_q, spec.block_k
    bi = spec.block_indices.numpy()
    total = 0
    for g in range(Hkv):
        r = 0
        for L in lens:
            nqb = (L + bq - 1) // bq
            for qb in range(nqb):
                blocks = set(int(b) for b in bi[g, r] if b >= 0)
                qi = np.arange(qb * bq, min(qb * bq + bq, L))
                for b in blocks:
                    kj = np.arange(b * bk, min(b * bk + bk, L))
                    if spec.causal and spec.window <= 0:
                        # count kj <= qi in closed form per row
                        total += int(np.clip(qi[:, None] - kj[None, :] >= 0, 0, 1).sum()) \
                            if b == qb else (len(qi) * len(kj) if b < qb else 0)
                    else:
                        vis = np.ones((len(qi), len(kj)), dtype=bool)
                        if spec.causal:
                            vis &= kj[None, :] <= qi[:, None]
                        if spec.window > 0:
                            vis &= (kj[None, :] < spec.n_sink) | (qi[:, None] - kj[None, :] < spec.window)
                        total += int(vis.sum())
                r += 1
    return int(total) * G


def gate_inputs(T_tot: int, Hq: int, seed: int):
    """Seeded per-(token, head) float32 arrays for the gate statistics and the
    gate-gradient backward: (values uniform in [0, 1) shaped like sink_s,
    standard-normal upstream gradients of sink_s)."""
    gen = _gen(seed)
    vals = torch.rand(T_tot, Hq, generator=gen, dtype=torch.float32)
    grads = torch.randn(T_tot, Hq, generator=gen, dtype=torch.float32)
    return vals, grads


def fp8_window_cache(d: DecodeInputs, seed: int):
    """A mixed-precision copy of a decode input's cache: the n_sink sink slots
    as they are, the window slots as FP8 E4M3 codes (uint8) of the values
    divided by a per-KV-head scale (float32 [Hkv], drawn so that the scaled
    values use the format's range).  Returns (k_sink, v_sink, k_codes, v_codes,
    k_scale, v_scale)."""
    gen = _gen(seed)
    Hkv = d.k_cache.shape[2]
    k_scale = (torch.rand(Hkv, generator=gen) * 0.05 + 0.02).float()
    v_scale = (torch.rand(Hkv, generator=gen) * 0.05 + 0.02).float()
    ns = d.n_sink

    def codes(x, sc):
        # torch's float8 cast does not saturate (|v| > 448 would become the
        # NaN code), so the scaled values are clamped to the format's range
        v = (x[:, ns:].float() / sc[None, None, :, None]).clamp(-448.0, 448.0)
        c = v.to(torch.float8_e4m3fn).view(torch.uint8)
        assert not bool(((c & 0x7F) == 0x7F).any()), "NaN code in the generated window cache"
        return c

    return (d.k_cache[:, :ns].clone(), d.v_cache[:, :ns].clone(), codes(d.k_cache, k_scale),
            codes(d.v_cache, v_scale), k_scale, v_scale)
