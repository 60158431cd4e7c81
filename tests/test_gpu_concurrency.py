"""Layers running at the same time on different streams share no device
state: each forward, launched while the other stream's forwards are in
flight, gives the bits it gives alone (the library keeps every intermediate
in the caller's workspace; its scratch-free entry points hold nothing
between calls)."""

import pytest
import torch

from mixture_experts_layer_51_b200 import moe as M
from mixture_experts_layer_51_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

PAIRS = [
    (WORKLOADS["top2_bf16"].replace(T=3000, d=512, H=768),
     WORKLOADS["openmoe_skew_bf16"].replace(T=4000, d=256, H=512, seq_len=1000)),
    (WORKLOADS["finegrained_bf16"].replace(T=2500, d=256, H=384),
     WORKLOADS["switch_tiny_fp32"]),
]


def _layer(w):
    t = make_inputs(w, "cuda")
    return M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act), t["x"]


@pytest.mark.parametrize("pair", range(len(PAIRS)))
def test_two_streams_give_the_bits_of_one(pair):
    (la, xa), (lb, xb) = (_layer(w) for w in PAIRS[pair])
    ya_ref, yb_ref = la(xa).clone(), lb(xb).clone()
    torch.cuda.synchronize()
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    sa.wait_stream(torch.cuda.current_stream())
    sb.wait_stream(torch.cuda.current_stream())
    ya, yb = torch.empty_like(ya_ref), torch.empty_like(yb_ref)
    for _ in range(4):
        # both streams' forwards in flight at once; each stream's own
        # forwards are in order, so its workspace is reused safely
        la(xa, y=ya, stream=sa)
        lb(xb, y=yb, stream=sb)
    torch.cuda.synchronize()
    assert torch.equal(ya, ya_ref)
    assert torch.equal(yb, yb_ref)
