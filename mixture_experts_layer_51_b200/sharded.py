"""One MoE layer over a batch whose tokens are split by position across ranks.

Expert capacity is a property of the whole batch ("How do Mixture of Expert
Models Work?", "Expert Capacity": C = ceil(cf * T * k / E) for the batch of
T tokens), and overflow is dropped by position ("Take a Closer Look at the
MoE LLM Routing", "Drop-towards-the-End").  When rank r holds the r-th
contiguous range of positions, the only cross-rank fact a rank needs is how
many assignments the lower-position ranks routed to each expert: E int32 per
rank, exchanged with one all-gather.  Each rank then keeps its i-th
assignment at expert e iff prior[e] + i < C, which is exactly what the
unsharded layer keeps.  Everything else (router, permutation, expert FFNs,
combine) is local to the rank's tokens.

The counts, the prefix over ranks and every compute step are libmoe.so
kernels (through the binding in ``moe``); torch.distributed only moves the
E-element count vectors.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import moe as M


def gather_expert_counts(counts, group=None):
    """All ranks' per-expert counts, stacked in rank order ([world, E] int32).

    NCCL gathers into one flat tensor; other backends (gloo, for host-side
    tests) use the list form."""
    world = dist.get_world_size(group)
    E = counts.numel()
    if dist.get_backend(group) == "nccl":
        out = torch.empty(world * E, dtype=counts.dtype, device=counts.device)
        dist.all_gather_into_tensor(out, counts.contiguous(), group=group)
        return out.view(world, E)
    parts = [torch.empty_like(counts) for _ in range(world)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts)


def moe_forward_sharded(layer, x, global_tokens=None, group=None, stream=None):
    """The layer output for this rank's tokens x [T_r, d], with capacity and
    drops decided over the whole batch.

    layer: an ``moe.MoELayer`` (position priority; Batch Priority Routing
    ranks tokens over the whole batch and is not sharded here).
    global_tokens: tokens in the whole batch; default T_r * world (equal
    shards).  stream: the CUDA stream to run on (default: the current one).
    Every kernel, the all-gather and every allocation run on that one stream,
    which first waits for the caller's current stream (where x was made);
    the caller's stream then waits for it, and the returned tensors are
    recorded as used there.  Returns y [T_r, d] and a dict of the
    intermediates.
    """
    if layer.priority != "position":
        raise ValueError("sharded capacity supports position priority only")
    T, _ = x.shape
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    T_all = T * world if global_tokens is None else int(global_tokens)
    caller = torch.cuda.current_stream(x.device)
    s = caller if stream is None else stream
    if s != caller:
        s.wait_stream(caller)
    with torch.cuda.stream(s):
        idx, gate, _ = M.moe_route(x, layer.Wg, layer.bias, layer.k, gating=layer.gating,
                                   gate_scale=layer.gate_scale)
        counts = M.moe_expert_counts(idx, layer.E)
        gathered = gather_expert_counts(counts, group)
        prior = M.moe_rank_prefix(gathered, rank)
        C = M.moe_capacity(T_all, layer.E, layer.k, layer.cf)
        perm = M.moe_permute(x, idx, layer.E, layer.cf, prior=prior, capacity=C)
        h, o, dev_error = M.moe_grouped_ffn(perm["xp"], perm["offsets"], perm["kept_counts"],
                                            layer.W1, layer.W3, layer.W2, layer.act)
        y = M.moe_unpermute_combine(o, perm["pos"], gate, x.dtype)
    info = dict(idx=idx, gate=gate, prior=prior, capacity=C, dev_error=dev_error, **perm)
    if s != caller:
        caller.wait_stream(s)
        x.record_stream(s)
        for t in [y] + [v for v in info.values() if torch.is_tensor(v)]:
            t.record_stream(caller)
    return y, info
