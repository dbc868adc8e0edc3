"""Inputs whose scores keep growing along the keys, so that the kernels' lazy
rescale of the running output runs on most key tiles.

The online softmax keeps a reference maximum per row and moves it (scaling
the partial output and row sum by 2^(m_old - m_new)) only when a tile's
maximum exceeds it by more than 2^8.  With the seeded normal inputs of the
other tests the first visible tile almost always sets a maximum that later
tiles do not beat by that much, so that branch would go unexercised.  Here
every query points along one unit direction v and key t carries a component
along v that grows linearly with its position, so the scores rise by
`growth` log2 units per 128 keys (on top of a little noise): a 128-key tile
exceeds the previous maximum by about `growth`, and pairs of randomly chosen
64-key blocks by varying amounts, some past the threshold and some not.
Everything is compared with the float64 oracle on the same rounded inputs
(the values V stay normal)."""
import pytest
import torch

import oracle
from learnable_sink_b200 import sinkattn as S
from learnable_sink_b200 import workloads as W

from gpu_util import TOL, check_lse, check_status, dev, max_abs, np64, run_fwd

pytestmark = pytest.mark.gpu

LOG2E = 1.4426950408889634


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    S.clear_status()
    yield
    check_status()


def _direction(D, seed):
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(D, generator=g, dtype=torch.float64)
    return v / v.norm()


def _growing(inp, growth, seed=3):
    """Rewrite q and k of `inp` so that q . k_t ~ 2 b(t) with b growing by
    `growth` log2 units of score per 128 keys of the sequence."""
    T, Hq, Hkv, D = inp.shape
    v = _direction(D, seed)
    cu = inp.mask.cu_seqlens.tolist()
    pos = torch.zeros(T, dtype=torch.float64)
    for a, b in zip(cu[:-1], cu[1:]):
        pos[a:b] = torch.arange(b - a, dtype=torch.float64)
    b = growth * pos / 128.0 / (2.0 * inp.scale * LOG2E)
    q = 0.05 * inp.q.double() + 2.0 * v
    k = 0.05 * inp.k.double() + b[:, None, None] * v
    inp.q = q.to(inp.q.dtype)
    inp.k = k.to(inp.k.dtype)
    return inp


def _compare_fwd(inp, out, lse, ss):
    tol = TOL[inp.q.dtype]
    ro, rl, rs = oracle.fwd(inp.q, inp.k, inp.v, inp.sink, inp.scale, **inp.mask.oracle_kwargs())
    eo = max_abs(np64(out), ro)
    assert eo <= tol["o"], f"O max abs {eo:.3e}"
    check_lse(np64(lse), rl, tol["lse"])
    assert max_abs(np64(ss), rs) <= tol["ss"]


def _spec(cu, **kw):
    return W.MaskSpec(cu_seqlens=torch.tensor(cu, dtype=torch.int32), **kw)


DENSE = {
    # two 128-row query tiles per CTA, 128-key tiles
    "causal_D128_G4": dict(cu=[0, 700, 1100], Hq=8, Hkv=2, D=128, mask=dict(causal=True)),
    "causal_D64_G2": dict(cu=[0, 650], Hq=4, Hkv=2, D=64, mask=dict(causal=True)),
    # the band's sink-only first tile followed by the window's tiles
    "band_D128": dict(cu=[0, 1000], Hq=4, Hkv=2, D=128,
                      mask=dict(causal=True, n_sink=4, window=300)),
    "non_causal_D128_G1": dict(cu=[0, 300, 640], Hq=2, Hkv=2, D=128, mask=dict(causal=False)),
}


@pytest.mark.parametrize("growth", [9.0, 20.0])
@pytest.mark.parametrize("name", list(DENSE))
def test_forward_growing_scores(name, growth):
    cfg = dict(DENSE[name])
    mask = _spec(cfg.pop("cu"), **cfg.pop("mask"))
    T = int(mask.cu_seqlens[-1])
    inp = _growing(W.make_attn(name, T_tot=T, dtype=torch.bfloat16, mask=mask, seed=41, **cfg),
                   growth)
    out, lse, ss, m, plan = run_fwd(inp)
    _compare_fwd(inp, out, lse, ss)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("G,D", [(8, 64), (2, 64), (4, 128)])
def test_forward_block_sparse_growing_scores(G, D, dtype):
    # 64-key blocks staged in pairs; at D = 64 the score tiles of consecutive
    # pairs sit in staggered tensor-memory regions and a rescale waits for
    # the previous pair's PV
    cu = W.random_cu_seqlens(1500, 300, 800, 17)
    bi = W.random_block_indices(cu, 2, 64, 64, 6, 18, shuffle=True)
    mask = W.MaskSpec(causal=True, cu_seqlens=cu, block_indices=bi, block_q=64, block_k=64)
    inp = _growing(W.make_attn("bs", T_tot=int(cu[-1]), Hq=2 * G, Hkv=2, D=D, dtype=dtype,
                               mask=mask, seed=43), 9.0)
    out, lse, ss, m, plan = run_fwd(inp)
    _compare_fwd(inp, out, lse, ss)


@pytest.mark.parametrize("D", [64, 128])
def test_decode_growing_scores(D):
    # partially filled caches (no wrap): slot order is token order, so the
    # scores rise along each warp's 16-row pieces
    d = W.decode(B=6, n_sink=4, window=700, Hq=8, Hkv=2, D=D, seqlen_range=(1, 704))
    d.cache_seqlens = torch.tensor([1, 40, 200, 333, 650, 704], dtype=torch.int32)
    B, Sl, Hkv, _ = d.k_cache.shape
    v = _direction(D, 5)
    slot = torch.arange(Sl, dtype=torch.float64)
    b = 9.0 * slot / 128.0 / (2.0 * d.scale * LOG2E)
    d.q = (0.05 * d.q.double() + 2.0 * v).to(torch.bfloat16)
    d.k_cache = (0.05 * d.k_cache.double() + b[None, :, None, None] * v).to(torch.bfloat16)
    out, lse, ss = S.decode(dev(d.q), dev(d.k_cache), dev(d.v_cache), dev(d.cache_seqlens),
                            d.n_sink, d.window, dev(d.sink), scale=d.scale, num_splits=3)
    torch.cuda.synchronize()
    ro, rl, rs = oracle.decode(d.q, d.k_cache, d.v_cache, d.cache_seqlens, d.n_sink, d.window,
                               d.sink, d.scale)
    tol = TOL[torch.bfloat16]
    assert max_abs(np64(out), ro) <= tol["o"]
    check_lse(np64(lse), rl, tol["lse"])
    assert max_abs(np64(ss), rs) <= tol["ss"]
