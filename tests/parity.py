"""Shared parity protocol: run the CUDA path through the C ABI and compare
every stage with the fp64 oracle.

Routing near a tie can legitimately pick either expert, so each stage is
checked twice:
  * end to end -- expert indices must match the oracle's wherever the
    oracle's margin (k-th minus (k+1)-th logit) exceeds 1e-3;
  * teacher-forced -- the oracle's capacity/permutation step is fed the GPU's
    indices (counts, kept counts, offsets, positions and drops must then be
    bit-exact everywhere), and the oracle's expert FFNs and combine are fed
    the GPU's selection (y must then meet the tolerance on every token).
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from mixture_experts_layer_51_b200 import moe as M

NEAR_TIE = 1e-3
BF16_MAX_ABS = 2e-2
BF16_REL_FRO = 5e-3
FP32_REL_FRO = 1e-5
GATE_ABS = 1e-4


def errors(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    diff = got - want
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    nrm = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(diff)) / nrm if nrm > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_y_close(got, want, dtype, what="y"):
    max_abs, rel = errors(got, want)
    if dtype == "bf16":
        assert max_abs <= BF16_MAX_ABS and rel <= BF16_REL_FRO, (
            f"{what}: max_abs={max_abs:.3g} rel_fro={rel:.3g}")
    else:
        assert rel <= FP32_REL_FRO, f"{what}: rel_fro={rel:.3g} max_abs={max_abs:.3g}"
    return max_abs, rel


def to_np(t):
    return t.detach().to("cpu").numpy()


def run_gpu(w, inp, device="cuda", gating="topk_softmax", gate_scale=1.0, priority="position"):
    """moe_forward through the ABI; returns y and every intermediate (numpy)."""
    dev = torch.device(device)
    t = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}
    layer = M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act,
                       gating=gating, gate_scale=gate_scale, priority=priority)
    y, st = layer(t["x"], stats=True)
    torch.cuda.synchronize(dev)
    views = layer.intermediates(w.T)
    out = {k: to_np(v) for k, v in views.items() if k in (
        "idx", "gate", "margin", "pos", "counts", "kept_counts", "offsets", "dev_error",
        "order")}
    out["y"] = to_np(y.float())
    out["stats"] = st
    out["layer"] = layer
    out["views"] = views
    out["dev_inputs"] = t
    return out


def padded_offsets(kept_counts):
    off = [0]
    for c in kept_counts:
        off.append(off[-1] + (int(c) + M.MOE_ROW_ALIGN - 1) // M.MOE_ROW_ALIGN * M.MOE_ROW_ALIGN)
    return np.array(off)


def check_routing(g, logits, k, gating="topk_softmax", gate_scale=1.0):
    """Indices vs the oracle away from near-ties; gates vs the oracle's
    gates at the GPU's selection; returns the near-tie count."""
    idx_o, _, margin_o = oracle.top_k(logits, k)
    far = margin_o > NEAR_TIE
    assert (g["idx"][far] == idx_o[far]).all(), "routing differs away from a near-tie"
    gi = g["idx"].astype(np.int64)
    if gating == "topk_softmax":
        gate_tf = oracle.gating_softmax(np.take_along_axis(logits, gi, 1))
    else:
        gate_tf = oracle.gating_softmax_all(logits, gi)
    gate_tf = gate_tf * gate_scale
    assert np.abs(g["gate"] - gate_tf).max() <= GATE_ABS * max(1.0, gate_scale)
    if k < logits.shape[1]:
        assert np.abs(g["margin"][far] - margin_o[far]).max() <= 1e-3
    return int((~far).sum()), idx_o


def check_xp_rows(xp_view, x, want_pos, kept, chunk=1 << 16):
    """Every kept row of xp is a bit-exact copy of its token's x row, at the
    row the oracle's positions name.  x: a torch tensor (compared on xp's
    device, in chunks, so full-size buffers never reach the host) or a numpy
    array (small cases)."""
    tt, jj = np.nonzero(kept)
    rows = want_pos[tt, jj]
    if torch.is_tensor(x):
        x = x.to(xp_view.device)
        for a in range(0, tt.size, chunk):
            r = torch.as_tensor(rows[a:a + chunk], device=xp_view.device, dtype=torch.long)
            s = torch.as_tensor(tt[a:a + chunk], device=xp_view.device, dtype=torch.long)
            assert torch.equal(xp_view.index_select(0, r), x.index_select(0, s)), (
                f"xp rows {a}..{a + r.numel()} are not exact copies")
        return
    r = torch.as_tensor(rows, device=xp_view.device, dtype=torch.long)
    got = to_np(xp_view.index_select(0, r).float())
    assert np.array_equal(got, x[tt].astype(np.float32)), "xp rows are not exact copies"


def check_permutation(g, x_np, T, E, k, cf, xp_view=None, priority="position"):
    """Teacher-forced permutation: bit-exact against the oracle's capacity
    step run on the GPU's own indices (and, for priority routing, on the
    oracle's order of the GPU's own gates).  With xp_view, every kept row of
    xp is checked too (x_np: the layer input, numpy or torch)."""
    C = oracle.capacity(T, E, k, cf)
    order = None
    if priority == "gate" and C is not None:
        order = oracle.priority_order(g["gate"])
        assert (g["order"] == order).all(), "priority order differs"
    counts, kept_counts, rank, kept = oracle.assign_capacity(g["idx"], E, C, order)
    assert (g["counts"] == counts).all()
    assert (g["kept_counts"] == kept_counts).all()
    off = padded_offsets(kept_counts)
    assert (g["offsets"] == off).all()
    want_pos = np.where(kept, off[g["idx"]] + rank, -1)
    assert (g["pos"] == want_pos).all()
    if xp_view is not None and kept.any():
        check_xp_rows(xp_view, x_np, want_pos, kept)
    return kept, C


def full_parity(w, inp, check_xp=True, gating="topk_softmax", gate_scale=1.0,
                priority="position"):
    """Whole-batch parity for sizes the oracle runs in seconds."""
    g = run_gpu(w, inp, gating=gating, gate_scale=gate_scale, priority=priority)
    assert int(g["dev_error"][0]) == 0
    x_np = to_np(inp["x"].float())
    logits = oracle.router_logits(inp["x"], inp["Wg"], inp["bias"])
    near, idx_o = check_routing(g, logits, w.k, gating, gate_scale)
    kept, C = check_permutation(g, x_np, w.T, w.E, w.k, w.cf,
                                g["views"]["xp"] if check_xp else None, priority)
    y_tf, _ = oracle.moe_forward_tokens(inp["x"], logits, g["idx"], kept, inp["W1"], inp["W3"],
                                        inp["W2"], w.act, gating, gate_scale)
    # The absolute bound is stated for the unscaled layer; a gate scale
    # multiplies |y| (and its final bf16 rounding) by the same factor, so
    # both sides are compared in unscaled units.
    errs = assert_y_close(g["y"] / gate_scale, y_tf / gate_scale, w.dtype)
    if priority == "position" and (near == 0 or (g["idx"] == idx_o).all()):
        ref = oracle.moe_forward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"],
                                 inp["W2"], w.k, w.cf, w.act, gating, gate_scale)
        assert (g["idx"] == ref["idx"]).all()
        assert (g["kept_counts"] == ref["kept_counts"]).all()
        assert_y_close(g["y"] / gate_scale, ref["y"] / gate_scale, w.dtype, "y (end to end)")
    return g, dict(near_ties=near, max_abs=errs[0], rel_fro=errs[1])
