"""A forward captured as a CUDA graph (moe_forward_graph_*) gives the same
bits as the eager forward, reads x afresh at every launch, and keeps the
intermediates in the workspace like moe_forward."""

import pytest
import torch

from mixture_experts_layer_51_b200 import moe as M
from mixture_experts_layer_51_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "switch_tiny_fp32": (WORKLOADS["switch_tiny_fp32"], "position"),
    "top2_small": (WORKLOADS["top2_bf16"].replace(T=600, d=256, H=384), "position"),
    "openmoe_small_capacity": (WORKLOADS["openmoe_skew_bf16"].replace(T=1100, d=256, H=512,
                                                                      seq_len=275), "position"),
    "bpr_ragged": (Workload("g", T=333, d=136, E=6, k=3, H=200, act="swiglu", dtype="bf16",
                            cf=0.5, seed=31), "gate"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_graph_replay_matches_eager(name):
    w, priority = CASES[name]
    t = make_inputs(w, "cuda")
    eager = M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act,
                       priority=priority)
    graphed = M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act,
                         priority=priority)
    x = t["x"].clone()
    g = graphed.graph(x)
    y_ref = eager(t["x"])
    y = g.launch()
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    a, b = eager.intermediates(w.T), graphed.intermediates(w.T)
    for key in ("idx", "gate", "pos", "counts", "kept_counts", "offsets", "dev_error"):
        assert torch.equal(a[key], b[key]), key
    # new tokens in the same buffer: the next launch reads them
    x2 = make_inputs(w.replace(seed=w.seed + 100), "cuda")["x"]
    x.copy_(x2)
    for _ in range(3):
        g.launch()
    y_ref2 = eager(x2)
    torch.cuda.synchronize()
    assert torch.equal(g.y, y_ref2)
    assert not torch.equal(y_ref2, y_ref)
    g.close()


def test_graph_holds_the_forward_kernels():
    """The bf16 layer with a streaming router (E a multiple of 8, at most 64)
    is five kernels -- router (with the permutation's counting), placement
    and copy, the two GEMMs, the combine -- and one memset of the error flag;
    priority routing adds the gate-order kernels."""
    w = WORKLOADS["top2_bf16"].replace(T=600, d=256, H=384)
    t = make_inputs(w, "cuda")
    layer = M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act)
    g = layer.graph(t["x"])
    assert g.nodes() == (5, 1)
    g.close()
    w, priority = CASES["bpr_ragged"]
    t = make_inputs(w, "cuda")
    bpr = M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act,
                     priority=priority)
    g = bpr.graph(t["x"])
    nk, no = g.nodes()
    assert nk > 5 and no >= 1
    g.close()
