"""A batch split by position over ranks, with the capacity exchange.

On one GPU the ranks are emulated one after another: each shard's counts
come from moe_expert_counts, the "all-gather" is a stack of those counts, and
each shard then runs moe_rank_prefix, moe_permute (whole-batch capacity and
the prefix), the expert FFNs and the combine on its own tokens.  No kernel
waits on another shard's kernels.  The kept assignments must be bit-exact
with the unsharded batch's (oracle capacity step on the GPU's indices) and y
within the bf16 tolerance of the oracle.
"""

import socket

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_51_b200 import moe as M
from mixture_experts_layer_51_b200.workloads import WORKLOADS, Workload, make_inputs

from parity import assert_y_close, to_np

pytestmark = pytest.mark.gpu


def _run_shards(w, t, bounds):
    T, E, k = w.T, w.E, w.k
    C = M.moe_capacity(T, E, k, w.cf)
    shards = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        idx, gate, _ = M.moe_route(t["x"][a:b], t["Wg"], t["bias"], k)
        shards.append(dict(a=a, b=b, idx=idx, gate=gate, counts=M.moe_expert_counts(idx, E)))
    gathered = torch.stack([s["counts"] for s in shards])
    for r, s in enumerate(shards):
        s["prior"] = M.moe_rank_prefix(gathered, r)
        p = M.moe_permute(t["x"][s["a"]:s["b"]], s["idx"], E, w.cf, prior=s["prior"], capacity=C)
        h, o, err = M.moe_grouped_ffn(p["xp"], p["offsets"], p["kept_counts"], t["W1"], t["W3"],
                                      t["W2"], w.act)
        s.update(p, err=err, y=M.moe_unpermute_combine(o, p["pos"], s["gate"], t["x"].dtype))
    torch.cuda.synchronize()
    return C, gathered, shards


@pytest.mark.parametrize("name,bounds", [
    ("openmoe_skew_bf16", (0, 300, 300, 301, 1100)),  # an empty and a one-token shard
    ("mixtral_bf16", (0, 130, 260, 390, 520)),         # four equal shards
    ("top2_bf16", (0, 599, 600)),
])
def test_sharded_capacity_matches_whole_batch(name, bounds):
    base = {"openmoe_skew_bf16": dict(T=1100, d=256, H=512, seq_len=275),
            "mixtral_bf16": dict(T=520, d=512, H=640, cf=0.8),
            "top2_bf16": dict(T=600, d=256, H=384, cf=1.0)}[name]
    w = WORKLOADS[name].replace(**base)
    inp = make_inputs(w, "cpu")
    dev = torch.device("cuda")
    t = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}
    C, gathered, shards = _run_shards(w, t, bounds)
    assert C >= 0
    idx = np.concatenate([to_np(s["idx"]) for s in shards])
    gate = np.concatenate([to_np(s["gate"]) for s in shards])
    # the router is per token: sharding does not change its bits
    idx_w, gate_w, _ = M.moe_route(t["x"], t["Wg"], t["bias"], w.k)
    assert np.array_equal(idx, to_np(idx_w)) and np.array_equal(gate, to_np(gate_w))
    counts, _, _, kept = oracle.assign_capacity(idx, w.E, C)
    assert not kept.all()  # capacity binds, so the prefix matters
    prior = np.zeros(w.E, dtype=np.int64)
    for r, s in enumerate(shards):
        a, b = s["a"], s["b"]
        local = np.bincount(idx[a:b].reshape(-1), minlength=w.E)
        assert np.array_equal(to_np(gathered[r]), local)
        assert np.array_equal(to_np(s["prior"]), prior)
        c, kc, rank, kept_r = oracle.assign_capacity_shard(idx[a:b], w.E, C, prior)
        assert np.array_equal(kept_r, kept[a:b])
        assert np.array_equal(to_np(s["counts"]), c)
        assert np.array_equal(to_np(s["kept_counts"]), kc)
        off = [0]
        for v in kc:
            off.append(off[-1] + (int(v) + M.MOE_ROW_ALIGN - 1) // M.MOE_ROW_ALIGN * M.MOE_ROW_ALIGN)
        off = np.array(off)
        assert np.array_equal(to_np(s["offsets"]), off)
        want_pos = np.where(kept_r, off[idx[a:b]] + rank, -1)
        assert np.array_equal(to_np(s["pos"]), want_pos)
        assert int(s["err"].item()) == 0
        prior = prior + local
    y = np.concatenate([to_np(s["y"].float()) for s in shards])
    logits = oracle.router_logits(inp["x"], inp["Wg"], inp["bias"])
    y_ref, _ = oracle.moe_forward_tokens(inp["x"], logits, idx, kept, inp["W1"], inp["W3"],
                                         inp["W2"], w.act)
    assert_y_close(y, y_ref, w.dtype)
    # the unsharded layer on the same batch
    layer = M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act)
    y_all = to_np(layer(t["x"]).float())
    assert_y_close(y, y_all, w.dtype, "y vs unsharded")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("side_stream", [False, True])
def test_forward_sharded_single_rank_equals_forward(side_stream):
    """moe_forward_sharded over a one-rank NCCL group is the plain layer, on
    the current stream or on a side stream (whose kernels, gather and
    allocations must be ordered against the caller's stream)."""
    import torch.distributed as dist
    from mixture_experts_layer_51_b200.sharded import moe_forward_sharded
    w = Workload("shard1", T=700, d=128, E=8, k=2, H=256, act="swiglu", dtype="bf16", cf=1.0,
                 seed=5)
    inp = make_inputs(w, "cpu")
    dev = torch.device("cuda")
    t = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}
    layer = M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        side = torch.cuda.Stream() if side_stream else None
        y, info = moe_forward_sharded(layer, t["x"], stream=side)
        # read on the caller's stream without a device-wide synchronise
        y = y.clone()
        err = info["dev_error"].clone()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y_ref = layer(t["x"])
    torch.cuda.synchronize()
    assert info["capacity"] == M.moe_capacity(w.T, w.E, w.k, w.cf)
    assert int(err.item()) == 0
    assert torch.equal(y, y_ref)
