"""Helpers for the GPU parity tests: run the CUDA path through the binding,
run the oracle on the same rounded inputs, compare."""
import numpy as np
import torch

from learnable_sink_b200 import sinkattn as S

# Tolerances (fp32: max abs 1e-4 on O/LSE, 1e-3 relative on gradients;
# bf16 with fp32 accumulation: 2e-2 max abs on O, 1e-3 on LSE and sink_s,
# 2e-2 relative on dQ/dK/dV/dsink).  Relative = max|g - ref| / max|ref|.
TOL = {
    torch.float32: dict(o=1e-4, lse=1e-4, ss=1e-4, grad=1e-3),
    torch.bfloat16: dict(o=2e-2, lse=1e-3, ss=1e-3, grad=2e-2),
    # f16 keeps 3 more mantissa bits than bf16 (P, dS and the outputs are
    # rounded to it); the bounds are a quarter of bf16's for O and half for
    # the gradients
    torch.float16: dict(o=5e-3, lse=1e-3, ss=1e-3, grad=1e-2),
}


def dev(x):
    return None if x is None else x.cuda().contiguous()


def run_fwd(inp, plan=None):
    m = S.Mask.from_spec(inp.mask)
    T, Hq, Hkv, D = inp.shape
    plan = plan or S.Plan(T, Hq, Hkv, m)
    out, lse, ss = S.fwd(dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.sink), m, plan, scale=inp.scale)
    torch.cuda.synchronize()
    return out, lse, ss, m, plan


def run_bwd(inp, out, lse, m, plan):
    dq, dk, dv, dsink = S.bwd(dev(inp.q), dev(inp.k), dev(inp.v), out, dev(inp.dout), lse,
                              dev(inp.sink), m, plan, scale=inp.scale)
    torch.cuda.synchronize()
    return dq, dk, dv, dsink


def np64(t):
    return t.detach().float().cpu().double().numpy()


def max_abs(a, b, mask=None):
    d = np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))
    if mask is not None:
        d = d[mask]
    return float(d.max()) if d.size else 0.0


def rel_err(a, ref):
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.abs(ref).max())
    return max_abs(a, ref) / (den if den > 0 else 1.0)


def check_lse(got, ref, tol):
    """LSE compare: -inf rows must match exactly, finite rows within tol."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), "empty-row pattern differs"
    fin = np.isfinite(ref)
    err = max_abs(got, ref, fin)
    assert err <= tol, f"LSE max abs {err:.3e} > {tol}"
    return err


def check_status():
    code = S.get_status()
    S.clear_status()
    assert code == 0, f"device status {S.ERR_NAMES.get(code, code)}"


def read_plan(plan):
    """Decode a plan buffer into python structures for the bit-exact tests."""
    w = plan.buf.cpu().numpy().view(np.int32)
    hdr = dict(zip(["magic", "n_fwd", "n_bwd", "n_tiles", "tile", "kh_slots", "T_tot", "Hkv",
                    "n_seq", "cap_tiles", "cap_items", "cap_entries", "n_entries", "fingerprint",
                    "off_tile_base", "off_fwd_items", "off_fwd_order", "off_fwd_entries",
                    "off_bwd_items", "off_bwd_order", "off_bwd_entries", "off_bwd_cursor",
                    "total_words"], w[:23].tolist()))

    def lists(items_off, order_off, ent_off, n):
        items = w[items_off: items_off + 8 * hdr["cap_items"]].reshape(-1, 8)
        order = w[order_off: order_off + n]
        out = {}
        for idx in order.tolist():
            it = items[idx]
            tile_start, tile_len, seq_start, seq_len, kvh, eoff, elen, tg = it.tolist()
            ents = w[ent_off + eoff: ent_off + eoff + elen].tolist()
            out[(kvh, tg)] = dict(tile_start=tile_start, tile_len=tile_len, seq_start=seq_start,
                                  seq_len=seq_len, entries=ents, rank=None)
        lens = [items[i][6] for i in order.tolist()]
        return out, order, lens

    fwd, fwd_order, fwd_lens = lists(hdr["off_fwd_items"], hdr["off_fwd_order"],
                                     hdr["off_fwd_entries"], hdr["n_fwd"])
    bwd, bwd_order, bwd_lens = lists(hdr["off_bwd_items"], hdr["off_bwd_order"],
                                     hdr["off_bwd_entries"], hdr["n_bwd"])
    return hdr, fwd, bwd, fwd_lens, bwd_lens
