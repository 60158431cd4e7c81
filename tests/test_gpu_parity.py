"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle.

Small runs cover every stage on whole batches that still span several tiles
and ragged tails; the full-size runs use the layer shapes and the launch
configuration the benchmark times, checking every token's routing, the whole
permutation, every kept row of xp and every element of y.
"""

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_51_b200 import moe as M
from mixture_experts_layer_51_b200.workloads import WORKLOADS, Workload, make_inputs

from parity import (assert_y_close, check_permutation, check_routing, full_parity, run_gpu,
                    to_np)

pytestmark = pytest.mark.gpu

SMALL = {
    # the five layer families at sizes the oracle runs in a second or two
    "switch_tiny_fp32": WORKLOADS["switch_tiny_fp32"],
    "top2_bf16": WORKLOADS["top2_bf16"].replace(T=600, d=256, H=384),
    "mixtral_bf16": WORKLOADS["mixtral_bf16"].replace(T=520, d=512, H=640),
    "openmoe_skew_bf16": WORKLOADS["openmoe_skew_bf16"].replace(T=1100, d=256, H=512, seq_len=275),
    "finegrained_bf16": WORKLOADS["finegrained_bf16"].replace(T=700, d=256, H=384),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_parity(name):
    w = SMALL[name]
    inp = make_inputs(w, "cpu")
    g, info = full_parity(w, inp)
    print(name, info)


def test_full_switch_tiny_fp32():
    # The fp32 workload is small enough to check whole at its full size.
    w = WORKLOADS["switch_tiny_fp32"]
    g, info = full_parity(w, make_inputs(w, "cpu"))
    assert g["stats"].capacity == 80


@pytest.mark.parametrize("case", [
    dict(T=1, d=64, E=4, k=2, H=128),            # single token
    dict(T=33, d=128, E=8, k=2, H=256),          # ragged vs the 32-token chunk
    dict(T=300, d=136, E=6, k=3, H=200),         # E not a multiple of 8, d/H tails
    dict(T=257, d=64, E=1, k=1, H=128),          # one expert: dense FFN
    dict(T=129, d=64, E=4, k=4, H=128),          # k == E
    dict(T=400, d=192, E=3, k=1, H=72, act="gelu"),  # bf16 GELU, odd sizes
    dict(T=2000, d=128, E=16, k=2, H=256, cf=0.25),  # heavy dropping
    dict(T=513, d=64, E=64, k=8, H=64),          # many tiny experts
    dict(T=1703, d=320, E=24, k=3, H=128),       # W_g box wider than E (24 of 32), d % 256 != 0
    dict(T=9999, d=200, E=40, k=5, H=96),        # router tiles of 72 rows, ragged last range
    dict(T=21011, d=128, E=16, k=2, H=64, cf=1.0),  # two router tiles per range
    # fp32: the router counts when its 8-token blocks are the token ranges
    # (T <= 8 x SMs) and leaves it to the permutation otherwise
    dict(T=333, d=72, E=5, k=2, H=200, cf=1.0, dtype="fp32"),
    dict(T=2500, d=64, E=4, k=2, H=136, cf=1.25, act="gelu", dtype="fp32"),
])
def test_edge_shapes(case):
    act = case.pop("act", "swiglu")
    cf = case.pop("cf", 0.0)
    dtype = case.pop("dtype", "bf16")
    w = Workload("edge", act=act, dtype=dtype, cf=cf, seed=11, **case)
    full_parity(w, make_inputs(w, "cpu"))


def test_all_tokens_on_one_expert_with_capacity():
    w = Workload("skew", T=700, d=128, E=8, k=2, H=256, act="swiglu", dtype="bf16", cf=1.0,
                 seed=5)
    inp = make_inputs(w, "cpu")
    inp["bias"] = torch.tensor([40.0, 30.0] + [0.0] * 6)  # experts 0 and 1 win everywhere
    g, _ = full_parity(w, inp)
    C = oracle.capacity(w.T, w.E, w.k, w.cf)
    assert g["counts"][0] == w.T and g["kept_counts"][0] == C
    # drops are exactly the latest tokens
    assert (g["pos"][:C, 0] >= 0).all() and (g["pos"][C:, 0] == -1).all()


@pytest.mark.parametrize("E,k,dtype", [(8, 3, "bf16"), (16, 5, "bf16"), (32, 5, "bf16"),
                                       (64, 7, "bf16"), (6, 3, "bf16"), (4, 1, "fp32")])
def test_exact_logit_ties_keep_the_lower_expert(E, k, dtype):
    """Router columns duplicated in pairs: every token's logits come in
    exactly equal pairs (the same products summed in the same order), so with
    odd k the TopK boundary splits a pair for many tokens.  The pages' order
    is a stable descending sort (equal logits: lower expert first), so every
    token's experts, in slot order, must equal the oracle's -- ties are not
    excluded here.  Covers each router back end (E 8 and 16: mma.sync with a
    K-split; 32 and 64: tcgen05; 6: the clustered mma.sync router; fp32)."""
    w = Workload("ties", T=1000, d=256, E=E, k=k, H=64, act="swiglu", dtype=dtype, cf=0.0,
                 seed=41)
    inp = make_inputs(w, "cpu")
    Wg = inp["Wg"].clone()
    Wg[:, 1::2] = Wg[:, 0::2]
    inp["Wg"] = Wg
    g = run_gpu(w, inp)
    logits = oracle.router_logits(inp["x"], Wg, inp["bias"])
    idx_o, _, margin = oracle.top_k(logits, k)
    assert (margin == 0).sum() > w.T // 4, "the boundary should split a pair often"
    assert np.array_equal(g["idx"], idx_o)
    assert np.array_equal(g["margin"][margin == 0], margin[margin == 0])
    kept, _ = check_permutation(g, to_np(inp["x"].float()), w.T, w.E, w.k, w.cf,
                                g["views"]["xp"])
    y_tf, _ = oracle.moe_forward_tokens(inp["x"], logits, g["idx"], kept, inp["W1"], inp["W3"],
                                        inp["W2"], w.act)
    assert_y_close(g["y"], y_tf, w.dtype)


def test_upcycling_identity_on_gpu():
    """Identical experts: the layer equals the dense FFN (within bf16)."""
    w = Workload("upcycle", T=300, d=128, E=8, k=2, H=256, act="swiglu", dtype="bf16", cf=0.0,
                 seed=6)
    inp = make_inputs(w, "cpu")
    for key in ("W1", "W3", "W2"):
        inp[key] = inp[key][:1].expand_as(inp[key]).contiguous()
    g = run_gpu(w, inp)
    dense = oracle.expert_ffn(inp["x"], inp["W1"][0], inp["W3"][0], inp["W2"][0], "swiglu")
    assert_y_close(g["y"], dense, "bf16", "upcycled layer vs dense FFN")


@pytest.mark.parametrize("name,scale", [("mixtral_bf16", 4.0), ("finegrained_bf16", 1.0),
                                        ("switch_tiny_fp32", 4.0)])
def test_switch_order_gating_parity(name, scale):
    """Softmax-then-TopK gates (Switch order) with the E/k output scale."""
    w = SMALL[name]
    full_parity(w, make_inputs(w, "cpu"), gating="softmax_topk", gate_scale=scale)


def test_switch_order_upcycling_identity_on_gpu():
    """Uniform router, identical experts, Softmax-then-TopK with gate scale
    E/k: the layer equals the dense FFN (within bf16)."""
    w = Workload("upcycle_switch", T=300, d=128, E=8, k=2, H=256, act="swiglu", dtype="bf16",
                 cf=0.0, seed=6)
    inp = make_inputs(w, "cpu")
    inp["Wg"] = torch.zeros_like(inp["Wg"])
    for key in ("W1", "W3", "W2"):
        inp[key] = inp[key][:1].expand_as(inp[key]).contiguous()
    g = run_gpu(w, inp, gating="softmax_topk", gate_scale=w.E / w.k)
    np.testing.assert_allclose(g["gate"], 0.5, atol=1e-6)
    dense = oracle.expert_ffn(inp["x"], inp["W1"][0], inp["W3"][0], inp["W2"][0], "swiglu")
    assert_y_close(g["y"], dense, "bf16", "upcycled Switch-order layer vs dense FFN")


@pytest.mark.parametrize("name", ["openmoe_skew_bf16", "switch_tiny_fp32", "finegrained_bf16"])
def test_batch_priority_routing_parity(name):
    """Capacity served by descending largest gate (Batch Priority Routing):
    the device radix argsort equals the oracle's stable argsort of the same
    gates, and the permutation and output follow the oracle."""
    w = SMALL[name]
    if w.cf <= 0:
        w = w.replace(cf=0.5)
    full_parity(w, make_inputs(w, "cpu"), priority="gate")


def test_priority_order_ties_and_sizes():
    """moe_priority_order alone: repeated gate values (stable ties) and sizes
    around the 256-element sort block."""
    rng = np.random.default_rng(3)
    for T in (1, 255, 256, 257, 5000):
        g = rng.integers(0, 7, size=(T, 2)).astype(np.float32) / 8 + 0.125
        gate = torch.tensor(g, device="cuda")
        order = M.moe_priority_order(gate)
        torch.cuda.synchronize()
        assert np.array_equal(to_np(order), oracle.priority_order(g))


def test_deterministic_bitwise():
    w = SMALL["finegrained_bf16"]
    inp = make_inputs(w, "cpu")
    a = run_gpu(w, inp)
    b = run_gpu(w, inp)
    assert np.array_equal(a["y"], b["y"])
    assert np.array_equal(a["pos"], b["pos"])


def test_forward_host_matches_device_forward():
    w = SMALL["top2_bf16"]
    inp = make_inputs(w, "cpu")
    g = run_gpu(w, inp)
    t = g["dev_inputs"]
    y_host = M.moe_forward_host(inp["x"].pin_memory(), t["Wg"], t["bias"], t["W1"], t["W3"],
                                t["W2"], w.k, w.cf, w.act)
    assert np.array_equal(y_host.float().numpy(), g["y"])


@pytest.mark.parametrize("T,cf", [(3001, 0.0), (4096, 0.0), (3001, 1.0)])
def test_forward_host_chunked_matches_device_forward(T, cf):
    """Dropless batches of >= 2048 tokens go through the chunked, overlapped
    host path; per-token results must not change (bit-exact).  With a
    capacity the batch stays whole."""
    w = Workload("hostpipe", T=T, d=256, E=8, k=2, H=384, act="swiglu", dtype="bf16", cf=cf,
                 seed=9)
    inp = make_inputs(w, "cpu")
    g = run_gpu(w, inp)
    t = g["dev_inputs"]
    for _ in range(2):
        y_host = M.moe_forward_host(inp["x"].pin_memory(), t["Wg"], t["bias"], t["W1"], t["W3"],
                                    t["W2"], w.k, w.cf, w.act)
        assert np.array_equal(y_host.float().numpy(), g["y"])


@pytest.mark.parametrize("depth,gating,cf", [(2, "topk_softmax", 0.0), (3, "softmax_topk", 1.0),
                                             (1, "topk_softmax", 1.25)])
def test_streaming_pipeline_matches_device_forward(depth, gating, cf):
    """moe_pipeline_*: seven different host batches streamed through `depth`
    slots (copies of one overlapping the forward of another) give, batch by
    batch, the same bits as the device-resident forward."""
    w = Workload("stream", T=1500, d=256, E=8, k=2, H=384, act="swiglu", dtype="bf16", cf=cf,
                 seed=12)
    inp = make_inputs(w, "cuda")
    layer = M.MoELayer(inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], w.k, w.cf,
                       w.act, gating=gating)
    g = torch.Generator().manual_seed(3)
    xs = [torch.randn(w.T, w.d, generator=g).bfloat16().pin_memory() for _ in range(7)]
    want = [to_np(layer(x.cuda()).float()) for x in xs]
    torch.cuda.synchronize()
    pipe = M.Pipeline(layer, w.T, depth=depth)
    ys = [torch.empty_like(x).pin_memory() for x in xs]
    for i, x in enumerate(xs):
        slot = i % depth
        if i >= depth:
            pipe.wait(slot)
            assert np.array_equal(ys[i - depth].float().numpy(), want[i - depth])
        pipe.submit(slot, x, ys[i])
    for i in range(len(xs) - depth, len(xs)):
        pipe.wait(i % depth)
        assert np.array_equal(ys[i].float().numpy(), want[i])
    pipe.close()


def test_stage_entry_points_match_forward():
    """moe_route -> moe_permute -> moe_grouped_ffn -> moe_unpermute_combine
    called one by one give the same bits as moe_forward."""
    w = SMALL["openmoe_skew_bf16"]
    inp = make_inputs(w, "cpu")
    g = run_gpu(w, inp)
    t = g["dev_inputs"]
    idx, gate, margin = M.moe_route(t["x"], t["Wg"], t["bias"], w.k)
    p = M.moe_permute(t["x"], idx, w.E, w.cf)
    h, o, err = M.moe_grouped_ffn(p["xp"], p["offsets"], p["kept_counts"], t["W1"], t["W3"],
                                  t["W2"], w.act)
    y = M.moe_unpermute_combine(o, p["pos"], gate, t["x"].dtype)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(to_np(idx), g["idx"])
    assert np.array_equal(to_np(p["pos"]), g["pos"])
    assert np.array_equal(to_np(y.float()), g["y"])


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_grouped_ffn_against_oracle(act):
    """The tcgen05 grouped GEMM alone, on hand-made expert blocks (sizes that
    are not tile multiples, an empty expert, a one-row expert)."""
    torch.manual_seed(0)
    E, d, H = 5, 320, 392
    kept = [130, 0, 257, 1, 128]
    off = [0]
    for c in kept:
        off.append(off[-1] + (c + 127) // 128 * 128)
    rows = off[-1]
    xp = torch.randn(rows, d).bfloat16()
    W1 = (torch.randn(E, d, H) / d ** 0.5).bfloat16()
    W3 = (torch.randn(E, d, H) / d ** 0.5).bfloat16() if act == "swiglu" else None
    W2 = (torch.randn(E, H, d) / H ** 0.5).bfloat16()
    dev = torch.device("cuda")
    offs = torch.tensor(off, dtype=torch.int32, device=dev)
    kc = torch.tensor(kept, dtype=torch.int32, device=dev)
    h, o, err = M.moe_grouped_ffn(xp.to(dev), offs, kc, W1.to(dev),
                                  None if W3 is None else W3.to(dev), W2.to(dev), act)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    h = to_np(h.float())
    o = to_np(o.float())
    for e in range(E):
        r = slice(off[e], off[e] + kept[e])
        if kept[e] == 0:
            continue
        xr = xp[r]
        if act == "swiglu":
            h_ref = oracle.silu(xr.double().numpy() @ W1[e].double().numpy()) * (
                xr.double().numpy() @ W3[e].double().numpy())
        else:
            h_ref = oracle.gelu(xr.double().numpy() @ W1[e].double().numpy())
        # h is rounded to bf16 once: relative error <= 2^-8 per element.
        assert np.all(np.abs(h[r] - h_ref) <= 2.0 ** -8 * np.abs(h_ref) + 1e-6), f"h expert {e}"
        # o given the GPU's own h: fp32 accumulation, then one rounding to
        # bf16 (relative error <= 2^-8, as for h), plus the accumulation's
        # own error (the absolute term).
        o_ref = h[r].astype(np.float64) @ W2[e].double().numpy()
        bound = 2.0 ** -8 * np.abs(o_ref) + 1e-5 * np.abs(o_ref).max()
        assert np.all(np.abs(o[r] - o_ref) <= bound), f"o expert {e}"


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
@pytest.mark.parametrize("d,H", [(72, 200), (200, 136)])
def test_grouped_ffn_fp32_against_oracle(act, d, H):
    """The fp32 grouped FFN (CUDA cores) alone: K of 72 (a partial last K
    slab) and 200 (seven slabs through the four-stage ring), a partial last
    column tile, an empty expert, a one-row expert, blocks that end inside
    a 64-row tile."""
    torch.manual_seed(1)
    E = 5
    kept = [130, 0, 257, 1, 128]
    off = [0]
    for c in kept:
        off.append(off[-1] + (c + 127) // 128 * 128)
    rows = off[-1]
    xp = torch.randn(rows, d)
    W1 = torch.randn(E, d, H) / d ** 0.5
    W3 = torch.randn(E, d, H) / d ** 0.5 if act == "swiglu" else None
    W2 = torch.randn(E, H, d) / H ** 0.5
    dev = torch.device("cuda")
    offs = torch.tensor(off, dtype=torch.int32, device=dev)
    kc = torch.tensor(kept, dtype=torch.int32, device=dev)
    h, o, err = M.moe_grouped_ffn(xp.to(dev), offs, kc, W1.to(dev),
                                  None if W3 is None else W3.to(dev), W2.to(dev), act)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    h = to_np(h)
    o = to_np(o)
    for e in range(E):
        r = slice(off[e], off[e] + kept[e])
        if kept[e] == 0:
            continue
        x64 = xp[r].double().numpy()
        if act == "swiglu":
            h_ref = oracle.silu(x64 @ W1[e].double().numpy()) * (x64 @ W3[e].double().numpy())
        else:
            h_ref = oracle.gelu(x64 @ W1[e].double().numpy())
        # fp32 accumulation of K products of O(1) terms: a few 1e-7 relative
        # to the row's scale.
        scale_h = np.abs(h_ref).max()
        assert np.abs(h[r] - h_ref).max() <= 1e-5 * scale_h, f"h expert {e}"
        o_ref = h_ref @ W2[e].double().numpy()
        assert np.abs(o[r] - o_ref).max() <= 1e-5 * np.abs(o_ref).max(), f"o expert {e}"


# ------------------------------------------------------ full-size layers
FULL = ["top2_bf16", "mixtral_bf16", "openmoe_skew_bf16", "finegrained_bf16"]


def _cpu(inp):
    return {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in inp.items()}


def _whole_batch_y(w, g, cpu, logits, kept, gating="topk_softmax"):
    """Every element of y against the oracle fed the GPU's selection (all
    tokens; the oracle converts one expert's weights to fp64 at a time)."""
    y_ref, _ = oracle.moe_forward_tokens(cpu["x"], logits, g["idx"], kept, cpu["W1"],
                                         cpu["W3"], cpu["W2"], w.act, gating)
    return assert_y_close(g["y"], y_ref, w.dtype)


@pytest.mark.parametrize("name", FULL)
def test_full_size_layer(name):
    """The benchmark's shapes and launch configuration, whole batch: every
    token's routing (away from near-ties), the whole permutation and every
    kept xp row bit-exact, and every element of y within the tolerance."""
    w = WORKLOADS[name]
    inp = make_inputs(w, "cuda")
    g = run_gpu(w, inp)
    assert int(g["dev_error"][0]) == 0
    cpu = _cpu(inp)
    logits = oracle.router_logits(cpu["x"], cpu["Wg"], cpu["bias"])
    near, _ = check_routing(g, logits, w.k)
    kept, C = check_permutation(g, inp["x"], w.T, w.E, w.k, w.cf, g["views"]["xp"])
    max_abs, rel = _whole_batch_y(w, g, cpu, logits, kept)
    dropped = int((~kept).sum())
    print(f"{name}: near_ties={near} dropped={dropped} y elements={g['y'].size} "
          f"max_abs={max_abs:.3g} rel_fro={rel:.3g}")
    if w.cf > 0:
        # Drop-towards-the-End, reported by position inside each sequence.
        L = w.seq_len or w.T
        for label, p, span in (("batch position", np.arange(w.T), w.T),
                               ("position in sequence", np.arange(w.T) % L, L)):
            rate = [float((~kept[(p >= a) & (p < a + span // 8)]).mean())
                    for a in range(0, span, span // 8)]
            print(f"drop rate by {label} octile:", [round(r, 4) for r in rate])


def test_many_tiles_per_cta_pair():
    """Two experts with 8000 rows each: the up projection has 2 x 32 x 16 =
    1024 pair tiles and the down projection 2 x 32 x 4 = 256 on at most 74
    CTA pairs, so every pair runs several tiles -- the persistent tile loop,
    the flip between the two TMEM accumulators and the wrap of every barrier
    phase -- and each expert ends on a ragged 64-row tail.  Whole batch,
    every element."""
    w = Workload("many_tiles", T=8000, d=1024, E=2, k=2, H=2048, act="swiglu", dtype="bf16",
                 cf=0.0, seed=17)
    inp = make_inputs(w, "cuda")
    g = run_gpu(w, inp)
    assert int(g["dev_error"][0]) == 0
    cpu = _cpu(inp)
    logits = oracle.router_logits(cpu["x"], cpu["Wg"], cpu["bias"])
    check_routing(g, logits, w.k)
    kept, _ = check_permutation(g, inp["x"], w.T, w.E, w.k, w.cf, g["views"]["xp"])
    assert (g["kept_counts"] == w.T).all()
    max_abs, rel = _whole_batch_y(w, g, cpu, logits, kept)
    print(f"many_tiles: max_abs={max_abs:.3g} rel_fro={rel:.3g}")


@pytest.mark.parametrize("cf", [0.0, 1.0])
def test_largest_expert_count_and_top_k(cf):
    """E = 64 and k = 8 (the largest the library takes) on a 65536-token
    batch (524288 assignments): routing away from near-ties, the whole
    permutation and every kept xp row bit-exact, every element of y within
    the tolerance."""
    w = Workload("max", T=65536, d=512, E=64, k=8, H=256, act="swiglu", dtype="bf16", cf=cf,
                 seed=31, bias_var=0.5)
    inp = make_inputs(w, "cuda")
    g = run_gpu(w, inp)
    assert int(g["dev_error"][0]) == 0
    cpu = _cpu(inp)
    logits = oracle.router_logits(cpu["x"], cpu["Wg"], cpu["bias"])
    check_routing(g, logits, w.k)
    kept, C = check_permutation(g, inp["x"], w.T, w.E, w.k, w.cf, g["views"]["xp"])
    assert (C is None) == (cf == 0.0)
    max_abs, rel = _whole_batch_y(w, g, cpu, logits, kept)
    print(f"max E/k cf={cf}: max_abs={max_abs:.3g} rel_fro={rel:.3g}")


def test_batch_priority_routing_full_size_openmoe():
    """Batch Priority Routing on the full OpenMoE-shaped batch (16384 tokens,
    E = 32, capacity 1024): the device order equals the oracle's stable
    argsort of the device gates, every position and kept xp row is
    bit-exact, every element of y meets the tolerance, and the dropped
    tokens are the least important at every expert."""
    w = WORKLOADS["openmoe_skew_bf16"]
    inp = make_inputs(w, "cuda")
    g = run_gpu(w, inp, priority="gate")
    assert int(g["dev_error"][0]) == 0
    cpu = _cpu(inp)
    logits = oracle.router_logits(cpu["x"], cpu["Wg"], cpu["bias"])
    check_routing(g, logits, w.k)
    kept, C = check_permutation(g, inp["x"], w.T, w.E, w.k, w.cf, g["views"]["xp"],
                                priority="gate")
    assert not kept.all()
    prio = g["gate"][:, 0]
    for e in range(w.E):
        pk = prio[np.nonzero((g["idx"] == e) & kept)[0]]
        pd = prio[np.nonzero((g["idx"] == e) & ~kept)[0]]
        if pk.size and pd.size:
            assert pd.max() <= pk.min()
    max_abs, rel = _whole_batch_y(w, g, cpu, logits, kept)
    print(f"BPR openmoe: max_abs={max_abs:.3g} rel_fro={rel:.3g}")


def test_plain_read_probe_reads_every_byte():
    """moe_probe_stream_read (the measurement aid): its sink is the XOR of
    every 32-bit word of the buffer, so a read that skipped any 16 bytes
    (or read one twice) would show."""
    g = torch.Generator().manual_seed(5)
    for n in (16, 4096, (1 << 22) + 48):
        buf = torch.randint(-2**31, 2**31 - 1, (n // 4,), generator=g, dtype=torch.int32)
        sink = torch.zeros(1, dtype=torch.int32, device="cuda")
        M.moe_probe_stream_read(buf.cuda(), sink)
        torch.cuda.synchronize()
        want = np.bitwise_xor.reduce(buf.numpy().view(np.uint32))
        assert int(sink.item()) & 0xffffffff == int(want), n


def test_reversed_k_rounds_opt_in():
    """MOE_TC_SERPENTINE=1 (read once per process, so in a child): the down
    projection runs the K steps of every other round of a CTA pair in
    reverse.  The many-tiles layer (256 down-projection tiles on at most 74
    pairs: both orders) and the small layers still match the oracle."""
    import os
    import subprocess
    import sys
    import textwrap
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    script = textwrap.dedent("""
        import sys
        sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
        import test_gpu_parity as T
        T.test_many_tiles_per_cta_pair()
        for name in T.SMALL:
            T.test_small_layer_parity(name)
        print("REVERSED_K_OK")
    """).format(root=root, tests=os.path.join(root, "tests"))
    env = dict(os.environ, MOE_TC_SERPENTINE="1")
    r = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    assert "REVERSED_K_OK" in r.stdout
