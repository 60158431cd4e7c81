"""The bf16 layer's storage roundings fit the parity tolerance, on the CPU.

The CUDA path rounds three tensors to bf16 on the way (h before the down
projection, the expert outputs o, and y) and accumulates in fp32.  This
models those roundings in fp64 on top of the oracle's own steps and checks
that, for the workloads' distributions, the modelled y stays inside the
bf16 bounds the GPU parity tests use (max-abs 2e-2, relative Frobenius
5e-3) with room to spare for the fp32 accumulation order.  No GPU is used.
"""

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_51_b200.workloads import WORKLOADS, make_inputs

from parity import BF16_MAX_ABS, BF16_REL_FRO


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("name,sizes", [
    ("top2_bf16", dict(T=512, d=512, H=768)),
    ("mixtral_bf16", dict(T=256, d=1024, H=1536)),
    ("finegrained_bf16", dict(T=512, d=512, H=384)),
])
def test_bf16_roundings_fit_the_tolerance(name, sizes):
    w = WORKLOADS[name].replace(**sizes)
    inp = make_inputs(w, "cpu")
    x = inp["x"].double().numpy()
    logits = oracle.router_logits(inp["x"], inp["Wg"], inp["bias"])
    idx, sel, _ = oracle.top_k(logits, w.k)
    g = oracle.gating_softmax(sel)
    y_exact = np.zeros((w.T, w.d))
    y_model = np.zeros((w.T, w.d))
    for e in range(w.E):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        W1, W3, W2 = (inp[k][e].double().numpy() for k in ("W1", "W3", "W2"))
        h = oracle.silu(x[rows] @ W1) * (x[rows] @ W3)
        gate = g[rows, slots][:, None]
        np.add.at(y_exact, rows, gate * (h @ W2))
        np.add.at(y_model, rows, gate * _bf16(_bf16(h) @ W2))   # h, then o, rounded
    y_model = _bf16(y_model)                                      # y rounded once
    err = y_model - y_exact
    max_abs = np.abs(err).max()
    rel = np.linalg.norm(err) / np.linalg.norm(y_exact)
    print(name, f"max_abs={max_abs:.4f} rel_fro={rel:.2e}")
    assert max_abs <= 0.8 * BF16_MAX_ABS, max_abs
    assert rel <= 0.7 * BF16_REL_FRO, rel
