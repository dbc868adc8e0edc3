"""Pins for the float64 oracle (CPU only).

Each test ties the oracle to something other than itself: the worked examples
printed on the pages (tests/golden/*.json, each with its citation), closed
forms, invariants, finite differences, brute-force counts, and special cases
that reduce to a library routine (torch's scaled_dot_product_attention and
autograd in float64).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from learnable_sink_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def causal_mask(T):
    return dict(causal=True, cu_seqlens=np.array([0, T], dtype=np.int32))


# ---------------------------------------------------------------- worked examples

def _two_token_problem(sink_value=None):
    """Page 1, section 1: one query, two keys with weights 0.75 / 0.25.
    alpha = 1, D = 2: x_1 = ln 3, x_2 = 0 gives e^x = 3 : 1."""
    ex = golden("worked_example.json")
    T = 3
    q = np.zeros((T, 1, 2)); k = np.zeros((T, 1, 2)); v = np.zeros((T, 1, 2))
    q[2, 0] = [1.0, 0.0]
    k[0, 0] = [math.log(3.0), 0.0]
    k[1, 0] = [0.0, 0.0]
    v[0, 0] = ex["V"][0]
    v[1, 0] = ex["V"][1]
    # block size 1: query 2 selects keys {0, 1} only (its own key is left out)
    mask = dict(causal=True, cu_seqlens=np.array([0, T], dtype=np.int32),
                block_indices=np.array([[[0, 1, 2], [0, 1, -1], [0, 1, -1]]], dtype=np.int32),
                block_q=1, block_k=1)
    sink = None if sink_value is None else np.array([sink_value])
    return ex, q, k, v, sink, mask


def test_worked_example_plain_attention():
    ex, q, k, v, sink, mask = _two_token_problem()
    out, lse, ss = oracle.fwd(q, k, v, sink, 1.0, **mask)
    np.testing.assert_allclose(out[2, 0], ex["O_plain"], rtol=0, atol=1e-14)
    assert abs(lse[2, 0] - math.log(4.0)) < 1e-14          # Z = 3 + 1
    assert abs(ss[2, 0] - 1.0) < 1e-14                     # no sink: all mass real


def test_worked_example_with_sink():
    # s = Z / (Z + e^a) = 0.2 with Z = 4  =>  e^a = 16
    ex, q, k, v, sink, mask = _two_token_problem(sink_value=math.log(16.0))
    out, lse, ss = oracle.fwd(q, k, v, sink, 1.0, **mask)
    np.testing.assert_allclose(out[2, 0], ex["O_with_sink"], rtol=0, atol=1e-14)
    assert abs(ss[2, 0] - ex["s"]) < 1e-14
    assert abs(lse[2, 0] - math.log(20.0)) < 1e-14
    # per-token probabilities: read them off with one-hot value rows
    v1 = np.zeros((3, 1, 2)); v1[0, 0] = [1, 0]; v1[1, 0] = [0, 1]
    p, _, _ = oracle.fwd(q, k, v1, sink, 1.0, **mask)
    np.testing.assert_allclose(p[2, 0], ex["weights_with_sink"], atol=1e-14)
    assert abs(1.0 - p[2, 0].sum() - ex["p_sink"]) < 1e-14


def test_renormalisation_example():
    g = golden("renormalisation.json")
    before = np.array(g["probs_before"])
    T = 3
    q = np.zeros((T, 1, 3)); k = np.zeros((T, 1, 3)); v = np.zeros((T, 1, 3))
    q[2, 0, 0] = 1.0
    for j in range(3):
        k[j, 0, 0] = math.log(before[j])   # logits whose softmax is `before`
        v[j, 0, j] = 1.0                   # one-hot values expose probabilities
    cu = np.array([0, T], dtype=np.int32)
    p, _, _ = oracle.fwd(q, k, v, None, 1.0, causal=True, cu_seqlens=cu)
    np.testing.assert_allclose(p[2, 0], before, atol=1e-14)
    # drop the initial token: window of 2 recent keys, no sink tokens kept
    p2, _, _ = oracle.fwd(q, k, v, None, 1.0, causal=True, window=2, n_sink=0, cu_seqlens=cu)
    np.testing.assert_allclose(p2[2, 0], [0.0] + g["probs_after_removing_first"], atol=1e-14)


def test_softmax_domination_example():
    g = golden("softmax_domination.json")
    n = g["n_rest"] + 1
    q = np.zeros((n, 1, 1)); k = np.zeros((n, 1, 1)); v = np.zeros((n, 1, n))
    q[n - 1, 0, 0] = 1.0
    k[:, 0, 0] = g["scores_rest"]
    k[0, 0, 0] = g["scores_first"]
    v = np.zeros((n, 1, n))
    for j in range(n):
        v[j, 0, j] = 1.0
    q2 = np.zeros((n, 1, n)); q2[:, :, 0] = q[:, :, 0]
    k2 = np.zeros((n, 1, n)); k2[:, :, 0] = k[:, :, 0]
    p, _, _ = oracle.fwd(q2, k2, v, None, 1.0, **causal_mask(n))
    first = p[n - 1, 0, 0]
    assert first >= g["page_attention_first_at_least"]
    exact_rest = math.exp(-10) / (math.exp(10) + 99 * math.exp(-10))
    np.testing.assert_allclose(p[n - 1, 0, 1:], exact_rest, rtol=1e-12)
    assert abs(first - math.exp(10) / (math.exp(10) + 99 * math.exp(-10))) < 1e-13


# ------------------------------------------------------- library special cases

def _random_problem(T, Hq, Hkv, D, seed, sink=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, Hq, D)); k = rng.standard_normal((T, Hkv, D))
    v = rng.standard_normal((T, Hkv, D)); dout = rng.standard_normal((T, Hq, D))
    a = rng.standard_normal(Hq) if sink else None
    return q, k, v, a, dout


MASKS = {
    "causal": dict(causal=True, cu_seqlens=np.array([0, 37], dtype=np.int32)),
    "band": dict(causal=True, n_sink=2, window=5, cu_seqlens=np.array([0, 37], dtype=np.int32)),
    "varlen": dict(causal=True, cu_seqlens=np.array([0, 10, 23, 37], dtype=np.int32)),
    "varlen_band": dict(causal=True, n_sink=3, window=4,
                        cu_seqlens=np.array([0, 10, 23, 37], dtype=np.int32)),
}


def _block_sparse_mask(T=37, Hkv=2, seed=5):
    cu = torch.tensor([0, 10, 23, 37], dtype=torch.int32)
    bi = W.random_block_indices(cu, Hkv, 4, 4, 2, seed, shuffle=True)
    return dict(causal=True, cu_seqlens=cu.numpy(), block_indices=bi.numpy(),
                block_q=4, block_k=4)


def _sdpa_forward(q, k, v, a, scale, vis):
    """Library reference: torch SDPA (float64) over the keys plus one extra
    zero key/value whose additive bias is a_h; vis[g] is [T, T] bool."""
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    qh = q.permute(1, 0, 2)
    kh = k.permute(1, 0, 2).repeat_interleave(G, 0)
    vh = v.permute(1, 0, 2).repeat_interleave(G, 0)
    zero = torch.zeros(Hq, 1, D, dtype=torch.float64)
    k_aug = torch.cat([kh, zero], 1)
    v_aug = torch.cat([vh, zero], 1)
    bias = torch.stack([torch.where(torch.from_numpy(vis[h // G]).bool(),
                                    torch.tensor(0.0, dtype=torch.float64),
                                    torch.tensor(-math.inf, dtype=torch.float64))
                        for h in range(Hq)])
    if a is None:
        col = torch.full((Hq, T, 1), -math.inf, dtype=torch.float64)
    else:
        col = a.reshape(Hq, 1, 1).expand(Hq, T, 1)
    mask = torch.cat([bias, col], -1)
    out = F.scaled_dot_product_attention(qh[None], k_aug[None], v_aug[None],
                                         attn_mask=mask[None], scale=scale)[0]
    logits = scale * torch.matmul(qh, k_aug.transpose(1, 2)) + mask
    lse = torch.logsumexp(logits, -1)
    p_sink = torch.softmax(logits, -1)[..., T]
    return out.permute(1, 0, 2), lse.T, (1 - p_sink).T


def _vis_all(T, Hq, Hkv, mask):
    return [oracle.visible_dense(T, Hq, Hkv, g, **mask) for g in range(Hkv)]


@pytest.mark.parametrize("mname", list(MASKS) + ["block_sparse"])
@pytest.mark.parametrize("with_sink", [True, False])
def test_forward_matches_library_sdpa(mname, with_sink):
    T, Hq, Hkv, D = 37, 4, 2, 16
    mask = MASKS[mname] if mname != "block_sparse" else _block_sparse_mask()
    q, k, v, a, _ = _random_problem(T, Hq, Hkv, D, seed=1, sink=with_sink)
    scale = 1 / math.sqrt(D)
    out, lse, ss = oracle.fwd(q, k, v, a, scale, **mask)
    vis = _vis_all(T, Hq, Hkv, mask)
    ro, rl, rs = _sdpa_forward(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
                               None if a is None else torch.from_numpy(a), scale, vis)
    np.testing.assert_allclose(out, ro.numpy(), atol=1e-12)
    np.testing.assert_allclose(lse, rl.numpy(), atol=1e-12)
    np.testing.assert_allclose(ss, rs.numpy(), atol=1e-12)


@pytest.mark.parametrize("mname", ["causal", "varlen_band", "block_sparse"])
def test_backward_matches_library_autograd(mname):
    T, Hq, Hkv, D = 37, 4, 2, 16
    mask = MASKS[mname] if mname != "block_sparse" else _block_sparse_mask()
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=2)
    scale = 1 / math.sqrt(D)
    dq, dk, dv, dsink = oracle.bwd(q, k, v, a, dout, scale, **mask)
    tq, tk, tv, ta = (torch.from_numpy(x).requires_grad_() for x in (q, k, v, a))
    vis = _vis_all(T, Hq, Hkv, mask)
    out, _, _ = _sdpa_forward(tq, tk, tv, ta, scale, vis)
    (out * torch.from_numpy(dout)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dsink, ta.grad.numpy(), atol=1e-11)


# ------------------------------------------------------ finite differences

def test_gradients_match_central_differences():
    T, Hq, Hkv, D = 12, 4, 2, 4
    mask = dict(causal=True, n_sink=1, window=4, cu_seqlens=np.array([0, 5, 12], dtype=np.int32))
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=3)
    scale = 1 / math.sqrt(D)
    dq, dk, dv, dsink = oracle.bwd(q, k, v, a, dout, scale, **mask)

    def loss(q_, k_, v_, a_):
        o, _, _ = oracle.fwd(q_, k_, v_, a_, scale, **mask)
        return float((o * dout).sum())

    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("sink", a, dsink)):
        idxs = [np.unravel_index(int(f), arr.shape)
                for f in rng.choice(arr.size, size=min(arr.size, 12), replace=False)]
        for idx in idxs:
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = {"q": q, "k": k, "v": v, "sink": a}
            args_m = dict(args_p)
            args_p[name] = plus
            args_m[name] = minus
            fd = (loss(args_p["q"], args_p["k"], args_p["v"], args_p["sink"]) -
                  loss(args_m["q"], args_m["k"], args_m["v"], args_m["sink"])) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, np.abs(grad).max()), (name, idx, fd, grad[idx])


# ---------------------------------------------------------- closed forms

def test_gate_identities_and_dsink_closed_form():
    """Page 1 section 4: s = Z/(Z+e^a) = e^(L_orig - L_new) = 1 - p_sink =
    sigma(L_orig - a), O_new = s O_orig; page 4 section 5: G = sigma(LSE - sink)
    equals s; page 1 section 7: dsink = -sum_i Delta (1 - s) = -sum Delta p_sink."""
    T, Hq, Hkv, D = 40, 4, 2, 8
    mask = MASKS["varlen_band"] | dict(cu_seqlens=np.array([0, 17, 40], dtype=np.int32))
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=4)
    scale = 0.3
    o_new, l_new, s = oracle.fwd(q, k, v, a, scale, **mask)
    o_orig, l_orig, s_orig = oracle.fwd(q, k, v, None, scale, **mask)
    sig = 1 / (1 + np.exp(-(l_orig - a[None, :])))
    np.testing.assert_allclose(s, sig, atol=1e-13)
    np.testing.assert_allclose(s, np.exp(l_orig - l_new), atol=1e-13)
    np.testing.assert_allclose(s, 1 - np.exp(a[None, :] - l_new), atol=1e-13)
    np.testing.assert_allclose(o_new, s[..., None] * o_orig, atol=1e-13)
    np.testing.assert_allclose(s_orig, 1.0, atol=1e-14)
    # L_new = logaddexp(L_orig, a)
    np.testing.assert_allclose(l_new, np.logaddexp(l_orig, a[None, :]), atol=1e-13)
    _, _, _, dsink = oracle.bwd(q, k, v, a, dout, scale, **mask)
    delta = (dout * o_new).sum(-1)
    np.testing.assert_allclose(dsink, -(delta * (1 - s)).sum(0), atol=1e-12)
    np.testing.assert_allclose(dsink, -(delta * np.exp(a[None, :] - l_new)).sum(0), atol=1e-12)


# ------------------------------------------- gate gradient and gate statistics
# Page "Attention Sink and the native MoE in attention layers"
# (lvdousha26.github.io), sections 4-5: head importance is the mean gate, the
# balance loss is lam * N_h * CV(Imp)^2, and training through it needs the
# backward to accept an upstream gradient of the gate sink_s.

@pytest.mark.parametrize("mname", ["causal", "varlen_band", "block_sparse"])
def test_gate_gradient_matches_library_autograd(mname):
    """oracle.bwd with dss equals float64 autograd of
    sum(dout * O) + sum(dss * sink_s) through torch's softmax."""
    T, Hq, Hkv, D = 37, 4, 2, 16
    mask = MASKS[mname] if mname != "block_sparse" else _block_sparse_mask()
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=21)
    dss = np.random.default_rng(22).standard_normal((T, Hq))
    scale = 1 / math.sqrt(D)
    dq, dk, dv, dsink = oracle.bwd(q, k, v, a, dout, scale, dss=dss, **mask)
    tq, tk, tv, ta = (torch.from_numpy(x).requires_grad_() for x in (q, k, v, a))
    vis = _vis_all(T, Hq, Hkv, mask)
    out, _, ss = _sdpa_forward(tq, tk, tv, ta, scale, vis)
    ((out * torch.from_numpy(dout)).sum() + (ss * torch.from_numpy(dss)).sum()).backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dsink, ta.grad.numpy(), atol=1e-11)


def test_gate_gradient_central_differences():
    T, Hq, Hkv, D = 12, 4, 2, 4
    mask = dict(causal=True, n_sink=1, window=4, cu_seqlens=np.array([0, 5, 12], dtype=np.int32))
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=23)
    dss = np.random.default_rng(24).standard_normal((T, Hq)) * 3.0
    scale = 1 / math.sqrt(D)
    grads = oracle.bwd(q, k, v, a, dout, scale, dss=dss, **mask)

    def loss(args):
        o, _, s_ = oracle.fwd(args[0], args[1], args[2], args[3], scale, **mask)
        return float((o * dout).sum() + (s_ * dss).sum())

    eps = 1e-6
    rng = np.random.default_rng(1)
    base = [q, k, v, a]
    for which, grad in enumerate(grads):
        arr = base[which]
        for f in rng.choice(arr.size, size=min(arr.size, 10), replace=False):
            idx = np.unravel_index(int(f), arr.shape)
            pl = [x.copy() for x in base]; mi = [x.copy() for x in base]
            pl[which][idx] += eps
            mi[which][idx] -= eps
            fd = (loss(pl) - loss(mi)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, np.abs(grad).max()), (which, idx, fd)


def test_gate_gradient_sigmoid_closed_form():
    """With dout = 0 and dss = 1 the loss is sum sink_s = sum sigma(L_orig - a),
    so dsink_h = -sum_i s (1 - s) (the logistic derivative) and dV = 0."""
    T, Hq, Hkv, D = 30, 4, 2, 8
    mask = MASKS["varlen_band"] | dict(cu_seqlens=np.array([0, 13, 30], dtype=np.int32))
    q, k, v, a, _ = _random_problem(T, Hq, Hkv, D, seed=25)
    scale = 0.4
    _, _, s = oracle.fwd(q, k, v, a, scale, **mask)
    _, _, dv, dsink = oracle.bwd(q, k, v, a, np.zeros((T, Hq, D)), scale,
                                 dss=np.ones((T, Hq)), **mask)
    np.testing.assert_allclose(dsink, -(s * (1 - s)).sum(0), atol=1e-12)
    assert np.all(dv == 0)


def test_gate_gradient_zero_dss_is_plain_backward():
    T, Hq, Hkv, D = 37, 4, 2, 16
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=26)
    ref = oracle.bwd(q, k, v, a, dout, 0.25, **MASKS["band"])
    got = oracle.bwd(q, k, v, a, dout, 0.25, dss=np.zeros((T, Hq)), **MASKS["band"])
    for x, y in zip(ref, got):
        np.testing.assert_array_equal(x, y)


def test_gate_importance_closed_forms():
    """Imp is the per-head mean gate: rows of a constant gate give that
    constant; for keys that all score 0 (q = 0) the gate of a row that sees n
    keys is n / (n + e^a)."""
    ss = np.tile(np.array([0.25, 0.5, 1.0]), (7, 1))
    np.testing.assert_allclose(oracle.gate_importance(ss), [0.25, 0.5, 1.0], rtol=0, atol=0)
    T, Hq, Hkv, D = 9, 2, 1, 4
    q = np.zeros((T, Hq, D)); k = np.ones((T, Hkv, D)); v = np.ones((T, Hkv, D))
    a = np.array([0.0, math.log(2.0)])
    _, _, s = oracle.fwd(q, k, v, a, 1.0, **causal_mask(T))
    n = np.arange(1, T + 1)
    expect = [np.mean(n / (n + math.exp(ah))) for ah in a]
    np.testing.assert_allclose(oracle.gate_importance(s), expect, atol=1e-15)


def test_gate_aux_loss_closed_forms_and_gradient():
    # Imp = (1, 3): mean 2, population std 1, CV = 1/2 -> lam * 2 * 1/4
    loss, d = oracle.gate_aux_loss(np.array([1.0, 3.0]), lam=0.1)
    assert abs(loss - 0.05) < 1e-15
    # balanced heads: zero loss, zero gradient
    loss, d = oracle.gate_aux_loss(np.full(8, 0.3), lam=1.0)
    assert loss == 0.0 and np.all(np.abs(d) < 1e-15)
    # shared/routed form: the top-1 head (5.0) is shared -> routed (1, 3)
    loss, d = oracle.gate_aux_loss(np.array([1.0, 5.0, 3.0]), lam=0.1, n_shared=1)
    assert abs(loss - 0.05) < 1e-15 and d[1] == 0.0
    # gradient against central differences
    rng = np.random.default_rng(27)
    imp = rng.uniform(0.1, 1.0, 12)
    for m in (0, 3):
        _, d = oracle.gate_aux_loss(imp, lam=0.7, n_shared=m)
        for h in range(12):
            e = np.zeros(12); e[h] = 1e-7
            fd = (oracle.gate_aux_loss(imp + e, 0.7, m)[0] -
                  oracle.gate_aux_loss(imp - e, 0.7, m)[0]) / 2e-7
            assert abs(fd - d[h]) < 1e-6, (m, h, fd, d[h])


@pytest.mark.parametrize("mname", ["causal", "band", "varlen_band", "block_sparse"])
def test_vanilla_gate_is_one_minus_first_token_probability(mname):
    """sigma(LSE_not0 - x_0) equals 1 - P(k_0) of the sink-free softmax; P(k_0)
    is read from the oracle's forward with V one-hot on each sequence's first
    token (an independent route through the attention forward)."""
    T, Hq, Hkv, D = 37, 4, 2, 16
    mask = MASKS[mname] if mname != "block_sparse" else _block_sparse_mask()
    q, k, _, _, _ = _random_problem(T, Hq, Hkv, D, seed=31)
    scale = 0.7
    cu = mask["cu_seqlens"]
    v = np.zeros((T, Hkv, D))
    v[cu[:-1], :, 0] = 1.0
    o, lse, _ = oracle.fwd(q, k, v, None, scale, **mask)
    gate = oracle.gate_vanilla(q, k, scale, **mask)
    seen = np.isfinite(lse)
    np.testing.assert_allclose(gate[seen], 1.0 - o[..., 0][seen], atol=1e-12)
    assert np.all(gate[~seen] == 0.0)


def test_vanilla_gate_closed_forms():
    """q = 0: every visible key scores 0, so the first token holds 1/n of the
    mass and G = 1 - 1/n under a causal mask; the first token of a sequence
    sees only itself (G = 0); a band without sink tokens hides k_0 from
    queries past the window (G = 1)."""
    T, Hq, Hkv, D = 20, 2, 1, 8
    q = np.zeros((T, Hq, D)); k = np.random.default_rng(32).standard_normal((T, Hkv, D))
    cu = np.array([0, 8, 20], dtype=np.int32)
    gate = oracle.gate_vanilla(q, k, 1.0, causal=True, cu_seqlens=cu)
    for s in range(2):
        n = np.arange(1, cu[s + 1] - cu[s] + 1)
        np.testing.assert_allclose(gate[cu[s]:cu[s + 1]], (1 - 1 / n)[:, None].repeat(Hq, 1),
                                   atol=1e-15)
    q = np.random.default_rng(33).standard_normal((T, Hq, D))
    gate = oracle.gate_vanilla(q, k, 1.0, causal=True, window=3, cu_seqlens=cu)
    assert np.all(gate[cu[:-1]] == 0.0)
    for s in range(2):
        for i in range(cu[s], cu[s + 1]):
            if i - cu[s] >= 3:
                assert np.all(gate[i] == 1.0)


def test_relative_probabilities_unchanged_by_sink():
    T, Hq, Hkv = 9, 2, 1
    rng = np.random.default_rng(7)
    q = rng.standard_normal((T, Hq, 3)); k = rng.standard_normal((T, Hkv, 3))
    v = np.zeros((T, Hkv, T))
    for j in range(T):
        v[j, 0, j] = 1.0
    q2 = np.zeros((T, Hq, T)); q2[..., :3] = q
    k2 = np.zeros((T, Hkv, T)); k2[..., :3] = k
    a = np.array([0.7, -1.3])
    p_new, _, _ = oracle.fwd(q2, k2, v, a, 1.0, **causal_mask(T))
    p_old, _, _ = oracle.fwd(q2, k2, v, None, 1.0, **causal_mask(T))
    for i in range(T):
        for h in range(Hq):
            ratio = p_new[i, h, :i + 1] / p_old[i, h, :i + 1]
            np.testing.assert_allclose(ratio, ratio[0], rtol=1e-13)


def test_zero_sink_differs_from_none():
    """Page 1 section 4: learnable_sink = 0 still contributes e^0 = 1."""
    T, Hq, Hkv, D = 16, 2, 1, 4
    q, k, v, _, _ = _random_problem(T, Hq, Hkv, D, seed=8, sink=False)
    _, l0, s0 = oracle.fwd(q, k, v, np.zeros(Hq), 0.5, **causal_mask(T))
    _, ln, sn = oracle.fwd(q, k, v, None, 0.5, **causal_mask(T))
    np.testing.assert_allclose(np.exp(l0), np.exp(ln) + 1.0, rtol=1e-13)
    assert np.all(s0 < 1.0) and np.allclose(sn, 1.0)


@pytest.mark.parametrize("a", [-1e4, -80.0, -20.0, 0.0, 20.0, 80.0])
def test_extreme_sink_values(a):
    T, Hq, Hkv, D = 20, 2, 1, 8
    q, k, v, _, _ = _random_problem(T, Hq, Hkv, D, seed=9, sink=False)
    scale = 1 / math.sqrt(D)
    o, l, s = oracle.fwd(q, k, v, np.full(Hq, a), scale, **causal_mask(T))
    o0, l0, _ = oracle.fwd(q, k, v, None, scale, **causal_mask(T))
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l)) and np.all(np.isfinite(s))
    np.testing.assert_allclose(l, np.logaddexp(l0, a), atol=1e-12)
    np.testing.assert_allclose(o, (np.exp(l0 - l))[..., None] * o0, atol=1e-12)
    if a <= -80:
        np.testing.assert_allclose(o, o0, atol=1e-12)
    if a >= 80:
        assert np.abs(o).max() < 1e-20 and s.max() < 1e-20


def test_empty_visible_set():
    """A query that sees no key (block selection empty): O = 0; with a sink
    LSE = a, sink_s = 0; without a sink LSE = -inf; gradients stay finite."""
    T, Hq, Hkv, D = 4, 2, 1, 3
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=10)
    bi = np.array([[[0], [-1], [1], [0]]], dtype=np.int32)  # query block 1 sees nothing
    mask = dict(causal=True, cu_seqlens=np.array([0, T], dtype=np.int32),
                block_indices=bi, block_q=1, block_k=1)
    o, l, s = oracle.fwd(q, k, v, a, 0.5, **mask)
    assert np.all(o[1] == 0) and np.allclose(l[1], a) and np.all(s[1] == 0)
    o, l, s = oracle.fwd(q, k, v, None, 0.5, **mask)
    assert np.all(o[1] == 0) and np.all(np.isneginf(l[1])) and np.all(s[1] == 0)
    dq, dk, dv, _ = oracle.bwd(q, k, v, None, dout, 0.5, **mask)
    assert np.all(dq[1] == 0) and np.all(np.isfinite(dk)) and np.all(np.isfinite(dv))


# --------------------------------------------------------------- masks

def _band_count(L, n_sink, window):
    return sum(min(i + 1, window) + min(n_sink, max(0, i + 1 - window)) for i in range(L))


@pytest.mark.parametrize("L,n_sink,window", [(40, 4, 8), (40, 0, 1), (33, 5, 40), (50, 3, 3)])
def test_mask_counts_closed_form(L, n_sink, window):
    cu = np.array([0, L], dtype=np.int32)
    causal = oracle.visible_dense(L, 1, 1, 0, causal=True, cu_seqlens=cu)
    assert causal.sum() == L * (L + 1) // 2
    assert np.array_equal(causal, np.tril(np.ones((L, L), dtype=np.uint8)))
    band = oracle.visible_dense(L, 1, 1, 0, causal=True, n_sink=n_sink, window=window, cu_seqlens=cu)
    assert band.sum() == _band_count(L, n_sink, window)
    if window >= L:
        assert np.array_equal(band, causal)
    if n_sink == 0 and window == 1:
        assert np.array_equal(band, np.eye(L, dtype=np.uint8))


def test_varlen_mask_is_block_diagonal():
    cu = np.array([0, 7, 7, 20, 31], dtype=np.int32)  # includes an empty sequence
    vis = oracle.visible_dense(31, 1, 1, 0, causal=True, cu_seqlens=cu)
    assert vis.sum() == sum(l * (l + 1) // 2 for l in np.diff(cu))
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        assert vis[a:b, :a].sum() == 0 and vis[a:b, b:].sum() == 0


def test_block_selection_all_earlier_equals_causal():
    cu = torch.tensor([0, 30, 61], dtype=torch.int32)
    bi_all = W.random_block_indices(cu, 2, 8, 8, n_random=100, seed=0)  # all earlier + diag
    m = dict(causal=True, cu_seqlens=cu.numpy(), block_q=8, block_k=8)
    for g in range(2):
        full = oracle.visible_dense(61, 2, 2, g, block_indices=bi_all.numpy(), **m)
        plain = oracle.visible_dense(61, 2, 2, g, **m)
        assert np.array_equal(full, plain)
    diag = np.full((2, bi_all.shape[1], 1), -1, dtype=np.int32)
    r = 0
    for L in (30, 31):
        for qb in range((L + 7) // 8):
            diag[:, r, 0] = qb
            r += 1
    vis = oracle.visible_dense(61, 2, 2, 0, block_indices=diag, **m)
    expect = sum(min(8, L - 8 * b) * (min(8, L - 8 * b) + 1) // 2
                 for L in (30, 31) for b in range((L + 7) // 8))
    assert vis.sum() == expect


def test_varlen_sequences_are_independent():
    T, Hq, Hkv, D = 37, 4, 2, 8
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=11)
    cu = np.array([0, 10, 23, 37], dtype=np.int32)
    o, l, s = oracle.fwd(q, k, v, a, 0.4, causal=True, n_sink=2, window=6, cu_seqlens=cu)
    dq, dk, dv, dsink = oracle.bwd(q, k, v, a, dout, 0.4, causal=True, n_sink=2, window=6, cu_seqlens=cu)
    dsink_sum = np.zeros(Hq)
    for s0, s1 in zip(cu[:-1], cu[1:]):
        sl = slice(s0, s1)
        one = np.array([0, s1 - s0], dtype=np.int32)
        o1, l1, _ = oracle.fwd(q[sl], k[sl], v[sl], a, 0.4, causal=True, n_sink=2, window=6, cu_seqlens=one)
        np.testing.assert_allclose(o[sl], o1, atol=1e-14)
        np.testing.assert_allclose(l[sl], l1, atol=1e-14)
        g1 = oracle.bwd(q[sl], k[sl], v[sl], a, dout[sl], 0.4, causal=True, n_sink=2, window=6, cu_seqlens=one)
        np.testing.assert_allclose(dq[sl], g1[0], atol=1e-13)
        np.testing.assert_allclose(dk[sl], g1[1], atol=1e-13)
        dsink_sum += g1[3]
    np.testing.assert_allclose(dsink, dsink_sum, atol=1e-12)


def test_tile_states_causal_closed_form():
    L, t = 300, 64   # 5 query tiles, the last one ragged (44 rows)
    st = oracle.tile_states(L, 1, 1, t, t, causal=True, cu_seqlens=np.array([0, L], dtype=np.int32))
    nq = (L + t - 1) // t
    assert st.shape == (1, nq, nq)
    for a in range(nq):
        for b in range(nq):
            expect = 2 if b < a else (1 if b == a else 0)
            assert st[0, a, b] == expect, (a, b)


def test_tile_states_band():
    L, t, n_sink, window = 600, 64, 4, 128
    cu = np.array([0, L], dtype=np.int32)
    st = oracle.tile_states(L, 1, 1, t, t, causal=True, n_sink=n_sink, window=window, cu_seqlens=cu)
    vis = oracle.visible_dense(L, 1, 1, 0, causal=True, n_sink=n_sink, window=window, cu_seqlens=cu)
    nq = st.shape[1]
    for a in range(nq):
        for b in range(nq):
            blk = np.zeros((t, t), dtype=np.uint8)
            sub = vis[a * t:(a + 1) * t, b * t:(b + 1) * t]
            blk[:sub.shape[0], :sub.shape[1]] = sub
            rows = min(t, L - a * t)
            cnt = blk[:rows].sum()
            expect = 0 if cnt == 0 else (2 if cnt == rows * t else 1)
            assert st[0, a, b] == expect
    # closed-form spot checks: the sink tile is partial for every far query tile,
    # and a tile fully inside the window is full
    assert st[0, nq - 1, 0] == 1
    assert st[0, 5, 4] == 2


# -------------------------------------------------------------- decode

def _logical_positions(n, n_sink, window):
    return list(range(min(n, n_sink))) + list(range(max(n_sink, n - window), n))


def test_decode_equals_band_forward_last_row():
    rng = np.random.default_rng(12)
    B, Hq, Hkv, D, n_sink, window = 6, 4, 2, 8, 2, 6
    S = n_sink + window
    ns = [1, 2, 5, 8, 9, 23]   # partially filled, exactly full, wrapped
    q = rng.standard_normal((B, Hq, D))
    a = rng.standard_normal(Hq)
    kc = rng.standard_normal((B, S, Hkv, D)); vc = rng.standard_normal((B, S, Hkv, D))
    out, lse, ss = oracle.decode(q, kc, vc, np.array(ns, dtype=np.int32), n_sink, window, a, 0.35)
    for b, n in enumerate(ns):
        # rebuild the logical sequence; evicted positions get random K/V
        kl = rng.standard_normal((n, Hkv, D)); vl = rng.standard_normal((n, Hkv, D))
        for p in _logical_positions(n, n_sink, window):
            slot = p if p < n_sink else n_sink + (p - n_sink) % window
            kl[p] = kc[b, slot]; vl[p] = vc[b, slot]
        ql = np.zeros((n, Hq, D)); ql[n - 1] = q[b]
        o, l, s = oracle.fwd(ql, kl, vl, a, 0.35, causal=True, n_sink=n_sink, window=window,
                             cu_seqlens=np.array([0, n], dtype=np.int32))
        np.testing.assert_allclose(out[b], o[n - 1], atol=1e-13)
        np.testing.assert_allclose(lse[b], l[n - 1], atol=1e-13)
        np.testing.assert_allclose(ss[b], s[n - 1], atol=1e-13)


def test_decode_invariant_to_ring_rotation():
    rng = np.random.default_rng(13)
    Hq, Hkv, D, n_sink, window = 4, 1, 8, 3, 7
    S = n_sink + window
    q = rng.standard_normal((1, Hq, D)); a = rng.standard_normal(Hq)
    kc = rng.standard_normal((1, S, Hkv, D)); vc = rng.standard_normal((1, S, Hkv, D))
    n0 = 50
    ref = oracle.decode(q, kc, vc, np.array([n0], np.int32), n_sink, window, a, 0.4)
    for r in range(1, window + 1):
        kr, vr = kc.copy(), vc.copy()
        kr[0, n_sink:] = np.roll(kc[0, n_sink:], r, axis=0)
        vr[0, n_sink:] = np.roll(vc[0, n_sink:], r, axis=0)
        got = oracle.decode(q, kr, vr, np.array([n0 + r], np.int32), n_sink, window, a, 0.4)
        for x, y in zip(ref, got):
            np.testing.assert_allclose(x, y, atol=1e-13)


@pytest.mark.parametrize("mname", ["varlen_band", "block_sparse"])
def test_sampled_backward_equals_full_backward(mname):
    """The sampled-gradient routine (used at full sizes) reproduces the full
    explicit-Jacobian backward on every sampled row and key."""
    T, Hq, Hkv, D = 37, 4, 2, 16
    mask = MASKS[mname] if mname != "block_sparse" else _block_sparse_mask()
    q, k, v, a, dout = _random_problem(T, Hq, Hkv, D, seed=14)
    dq, dk, dv, _ = oracle.bwd(q, k, v, a, dout, 0.3, **mask)
    rng = np.random.default_rng(1)
    rows = np.stack([rng.integers(0, T, 20), rng.integers(0, Hq, 20)], 1)
    keys = np.stack([rng.integers(0, T, 15), rng.integers(0, Hkv, 15)], 1)
    sq, sk, sv = oracle.bwd_sampled(q, k, v, a, dout, 0.3, rows, keys, **mask)
    np.testing.assert_allclose(sq, dq[rows[:, 0], rows[:, 1]], atol=1e-13)
    np.testing.assert_allclose(sk, dk[keys[:, 0], keys[:, 1]], atol=1e-13)
    np.testing.assert_allclose(sv, dv[keys[:, 0], keys[:, 1]], atol=1e-13)


@pytest.mark.parametrize("mname", ["varlen_band", "block_sparse"])
def test_forward_rows_equal_full_forward_rows(mname):
    """fwd_rows (the row-sampled forward used on full-size inputs) returns
    exactly the full forward's values at the sampled (token, head) rows."""
    T, Hq, Hkv, D = 37, 4, 2, 16
    mask = MASKS[mname] if mname != "block_sparse" else _block_sparse_mask()
    q, k, v, a, _ = _random_problem(T, Hq, Hkv, D, seed=41)
    out, lse, ss = oracle.fwd(q, k, v, a, 0.3, **mask)
    rng = np.random.default_rng(42)
    rows = np.stack([rng.integers(0, T, 25), rng.integers(0, Hq, 25)], 1).astype(np.int32)
    ro, rl, rs = oracle.fwd_rows(q, k, v, a, 0.3, rows, **mask)
    np.testing.assert_array_equal(ro, out[rows[:, 0], rows[:, 1]])
    np.testing.assert_array_equal(rl, lse[rows[:, 0], rows[:, 1]])
    np.testing.assert_array_equal(rs, ss[rows[:, 0], rows[:, 1]])


# ------------------------------------------- mixed-precision (FP8 window) decode

def test_fp8_e4m3_values_match_the_library_conversion():
    """Every one of the 256 codes against torch's float8_e4m3fn conversion."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.fp8_e4m3_value(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    np.testing.assert_array_equal(got[~np.isnan(got)], ref[~np.isnan(ref)])


def test_fp8_e4m3_closed_forms():
    v = oracle.fp8_e4m3_value(np.array([0x38, 0x7E, 0x01, 0x08, 0xB8, 0x00, 0x80, 0x7F, 0xFF],
                                        dtype=np.uint8))
    np.testing.assert_array_equal(v[:7], [1.0, 448.0, 2.0 ** -9, 2.0 ** -6, -1.0, 0.0, -0.0])
    assert np.isnan(v[7]) and np.isnan(v[8])


def test_fp8_window_decode_is_the_decode_of_the_dequantised_cache():
    """The sink slots stay as given and the window slots are code value x
    per-KV-head scale: equal to the plain decode on that cache, and doubling
    one head's scale equals doubling that head's window rows."""
    d = W.decode(B=3, n_sink=4, window=28, Hq=8, Hkv=2, D=16, seqlen_range=(0, 90))
    d.cache_seqlens = torch.tensor([2, 17, 90], dtype=torch.int32)
    ks, vs, kc, vc, ksc, vsc = W.fp8_window_cache(d, 7)
    got = oracle.decode_fp8_window(d.q, ks, vs, kc, vc, ksc, vsc, d.cache_seqlens, d.n_sink,
                                   d.window, d.sink, d.scale)
    kw = torch.from_numpy(kc.numpy()).view(torch.float8_e4m3fn).double() * ksc.double()[None, None, :, None]
    vw = torch.from_numpy(vc.numpy()).view(torch.float8_e4m3fn).double() * vsc.double()[None, None, :, None]
    k = torch.cat([ks.double(), kw], 1)
    v = torch.cat([vs.double(), vw], 1)
    ref = oracle.decode(d.q, k, v, d.cache_seqlens, d.n_sink, d.window, d.sink, d.scale)
    for a, b in zip(got, ref):
        np.testing.assert_array_equal(a, b)
    ksc2 = ksc.clone()
    ksc2[1] *= 2
    got2 = oracle.decode_fp8_window(d.q, ks, vs, kc, vc, ksc2, vsc, d.cache_seqlens, d.n_sink,
                                    d.window, d.sink, d.scale)
    k2 = k.clone()
    k2[:, d.n_sink:, 1] *= 2
    ref2 = oracle.decode(d.q, k2, v, d.cache_seqlens, d.n_sink, d.window, d.sink, d.scale)
    for a, b in zip(got2, ref2):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-15)
    assert not np.allclose(got2[0], got[0])


def test_fp8_e4m3_encode_round_trips_every_code():
    """Every finite code's value encodes back to that code (both signs)."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.fp8_e4m3_value(codes)
    got = oracle.fp8_e4m3_encode(vals)
    # +0 and -0 are distinct codes with the same value: the sign bit decides
    assert np.array_equal(got, codes)


def test_fp8_e4m3_encode_matches_the_library_conversion_in_range():
    """Round to nearest, ties to even, against torch's float8_e4m3fn cast on
    values inside the format's range (where the cast does not saturate)."""
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.normal(0, 30, 20000), rng.uniform(-448, 448, 20000),
                        rng.normal(0, 1e-2, 5000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.fp8_e4m3_encode(x), ref)


def test_fp8_e4m3_encode_closed_forms():
    """Ties go to the even mantissa, magnitudes past 448 saturate, NaN keeps
    the NaN code, tiny values round to signed zero."""
    x = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 448.0, 464.0, 1e6, -1e6,
                  float("nan"), -1e-30, 0.0, -0.0])
    want = [0x38, 0x3A, 0x00, 0x02, 0x7E, 0x7E, 0x7E, 0xFE, 0x7F, 0x80, 0x00, 0x80]
    assert oracle.fp8_e4m3_encode(x).tolist() == want


def test_fp8_cache_append_slot_rule():
    """Positions below n_sink land in the bf16 sink slots unchanged; later
    positions land in window row (p - n_sink) mod window as codes of
    value / scale; a sequence with no token writes nothing."""
    B, Hkv, D, ns, win = 3, 2, 4, 2, 5
    kn = np.arange(B * Hkv * D, dtype=np.float64).reshape(B, Hkv, D) / 8.0
    vn = -kn
    ks = np.zeros((B, ns, Hkv, D))
    kw = np.zeros((B, win, Hkv, D), dtype=np.uint8)
    sc = np.array([0.5, 0.25], dtype=np.float32)
    cs = np.array([2, 0, 9], dtype=np.int32)  # positions 1, none, 8
    k2, v2, kw2, vw2 = oracle.cache_append_fp8(kn, vn, cs, ks, ks, kw, kw, sc, sc, ns, win)
    assert np.array_equal(k2[0, 1], kn[0]) and np.array_equal(v2[0, 1], vn[0])
    assert not k2[1].any() and not kw2[1].any()
    r = (8 - ns) % win
    assert np.array_equal(kw2[2, r], oracle.fp8_e4m3_encode(kn[2] / sc[:, None]))
    # within half a grid step (1/16 relative for normal values) of the value
    back = oracle.fp8_e4m3_value(kw2[2, r]) * sc[:, None]
    assert np.all(np.abs(back - kn[2]) <= np.abs(kn[2]) / 16 + 1e-12)
    assert np.count_nonzero(kw2.reshape(B, win, -1).any(axis=2)) == 1
