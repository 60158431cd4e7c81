"""GPU parity of expert-choice routing (through the C ABI) against the oracle.

The selection is decided by fp32 affinities on the GPU and fp64 ones in the
oracle, so it is checked twice, like token choice:
  * teacher-forced -- the oracle's selection rule run on the GPU's own fp32
    affinities must give exactly the GPU's tokens, rows and positions, and
    the oracle layer weighted by those affinities must match y;
  * end to end -- affinities within 2e-5 of the oracle's, and the choice
    identical wherever the oracle's affinity is more than 1e-4 away from
    that expert's cut-off.
"""

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_51_b200 import moe as M
from mixture_experts_layer_51_b200.workloads import WORKLOADS, Workload, make_inputs

from parity import assert_y_close, to_np

pytestmark = pytest.mark.gpu

SCORE_ABS = 2e-5
NEAR_CUT = 1e-4

CASES = {
    "top2_bf16": WORKLOADS["top2_bf16"].replace(T=600, d=256, H=384, cf=1.0),
    "mixtral_bf16": WORKLOADS["mixtral_bf16"].replace(T=520, d=512, H=640, cf=1.0),
    "finegrained_bf16": WORKLOADS["finegrained_bf16"].replace(T=700, d=256, H=384, cf=1.0),
    "openmoe_skew_bf16": WORKLOADS["openmoe_skew_bf16"].replace(T=1100, d=256, H=512,
                                                                seq_len=275),
    "switch_tiny_fp32": WORKLOADS["switch_tiny_fp32"],
    "room_for_all": Workload("room", T=100, d=64, E=4, k=2, H=128, act="swiglu", dtype="bf16",
                             cf=8.0, seed=21),
    "one_token": Workload("one", T=1, d=64, E=4, k=2, H=64, act="swiglu", dtype="bf16",
                          cf=1.0, seed=22),
    "ragged_gelu": Workload("rg", T=333, d=136, E=6, k=3, H=200, act="gelu", dtype="bf16",
                            cf=0.5, seed=23),
}


def _run(w, inp):
    dev = torch.device("cuda")
    t = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}
    layer = M.ExpertChoiceLayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act)
    y, st = layer(t["x"], stats=True)
    torch.cuda.synchronize()
    views = layer.intermediates(w.T)
    return t, layer, y, st, views


def _check(w, inp):
    t, layer, y, st, v = _run(w, inp)
    n = M.moe_expert_choice_tokens(w.T, w.E, w.k, w.cf)
    assert n == min(w.T, oracle.capacity(w.T, w.E, w.k, w.cf))
    assert st.device_error == 0 and v["n"] == n
    S_gpu = to_np(v["scores"]).T.astype(np.float64)
    pos = to_np(v["pos"])
    tok = to_np(v["tok"])
    # teacher-forced selection: bit-exact
    sel, tokens = oracle.expert_choice_select(S_gpu, n)
    assert np.array_equal(pos >= 0, sel)
    npad = (n + 127) // 128 * 128
    for e in range(w.E):
        assert np.array_equal(tok[e], tokens[e])
        assert np.array_equal(pos[tokens[e], e], e * npad + np.arange(n))
    assert np.array_equal(to_np(v["kept_counts"]), np.full(w.E, n))
    assert np.array_equal(to_np(v["offsets"]), np.arange(w.E + 1) * npad)
    # the gathered rows are exact copies
    x_np = to_np(inp["x"].float())
    if n > 0:
        xp = to_np(v["xp"].float())
        for e in range(w.E):
            assert np.array_equal(xp[e * npad:e * npad + n], x_np[tokens[e]])
    # end to end: affinities and the choice away from each expert's cut-off
    logits = oracle.router_logits(inp["x"], inp["Wg"], inp["bias"])
    S_o = oracle.expert_choice_scores(logits)
    assert np.abs(S_gpu - S_o).max() <= SCORE_ABS
    sel_o, _ = oracle.expert_choice_select(S_o, n)
    if 0 < n < w.T:
        cut = np.sort(S_o, axis=0)[::-1][n - 1]       # n-th largest per expert
        far = np.abs(S_o - cut[None, :]) > NEAR_CUT
        assert np.array_equal(sel[far], sel_o[far])
    # y against the oracle weighted by the GPU's affinities
    ref = oracle.moe_forward_expert_choice(inp["x"], inp["Wg"], inp["bias"], inp["W1"],
                                           inp["W3"], inp["W2"], w.k, w.cf, w.act, scores=S_gpu)
    assert np.array_equal(ref["sel"], sel)
    errs = assert_y_close(to_np(y.float()), ref["y"], w.dtype)
    return t, layer, y, dict(max_abs=errs[0], rel_fro=errs[1], uncovered=int((~sel.any(1)).sum()))


@pytest.mark.parametrize("name", list(CASES))
def test_expert_choice_parity(name):
    w = CASES[name]
    _, _, _, info = _check(w, make_inputs(w, "cpu"))
    print(name, info)


def test_expert_choice_stage_entry_points_match_forward():
    w = CASES["finegrained_bf16"]
    inp = make_inputs(w, "cpu")
    t, layer, y, _ = _check(w, inp)
    n = M.moe_expert_choice_tokens(w.T, w.E, w.k, w.cf)
    S = M.moe_expert_choice_route(t["x"], t["Wg"], t["bias"])
    s = M.moe_expert_choice_select(S, n)
    xp = M.moe_expert_choice_permute(t["x"], s["pos"], n)
    h, o, err = M.moe_grouped_ffn(xp, s["offsets"], s["kept_counts"], t["W1"], t["W3"], t["W2"],
                                  w.act)
    y2 = M.moe_expert_choice_combine(o, s["pos"], S, t["x"].dtype)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    v = layer.intermediates(w.T)
    assert torch.equal(S, v["scores"]) and torch.equal(s["pos"], v["pos"])
    assert torch.equal(y2, y)


def test_expert_choice_uniform_router_on_gpu():
    """W_g = 0: equal affinities 1/E, so every expert takes tokens 0..n-1
    (ties to the lower position); with identical experts y_t = FFN(x_t) for
    those tokens and 0 for the rest."""
    w = Workload("ecu", T=300, d=128, E=4, k=1, H=256, act="swiglu", dtype="bf16", cf=1.0,
                 seed=24)
    inp = make_inputs(w, "cpu")
    inp["Wg"] = torch.zeros_like(inp["Wg"])
    for key in ("W1", "W3", "W2"):
        inp[key] = inp[key][:1].repeat(w.E, 1, 1).contiguous()
    t, layer, y, st, v = _run(w, inp)
    n = M.moe_expert_choice_tokens(w.T, w.E, w.k, w.cf)
    assert n == 75
    tok = to_np(v["tok"])
    assert all(np.array_equal(tok[e], np.arange(n)) for e in range(w.E))
    dense = oracle.expert_ffn(inp["x"][:n], inp["W1"][0], inp["W3"][0], inp["W2"][0], "swiglu")
    yn = to_np(y.float())
    assert_y_close(yn[:n], dense, "bf16")
    assert (yn[n:] == 0).all()


def test_expert_choice_deterministic_bitwise():
    w = CASES["openmoe_skew_bf16"]
    inp = make_inputs(w, "cpu")
    t, layer, y1, _, _ = _run(w, inp)
    y2 = layer(t["x"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_expert_choice_full_size_selection():
    """The fine-grained layer shape at full size (T = 16384, E = 64): the
    selection against the oracle's rule on the GPU's affinities, bit-exact,
    and a sample of tokens' outputs."""
    w = WORKLOADS["finegrained_bf16"].replace(cf=1.0)
    inp = make_inputs(w, "cpu")
    t, layer, y, st, v = _run(w, inp)
    assert st.device_error == 0
    n = M.moe_expert_choice_tokens(w.T, w.E, w.k, w.cf)
    S_gpu = to_np(v["scores"]).T.astype(np.float64)
    sel, tokens = oracle.expert_choice_select(S_gpu, n)
    pos = to_np(v["pos"])
    assert np.array_equal(pos >= 0, sel)
    rng = np.random.default_rng(0)
    sample = np.sort(rng.choice(w.T, 48, replace=False))
    ys = np.zeros((sample.size, w.d))
    x = inp["x"]
    for e in range(w.E):
        rows = np.nonzero(sel[sample, e])[0]
        if rows.size == 0:
            continue
        out = oracle.expert_ffn(x[sample[rows]], inp["W1"][e], inp["W3"][e], inp["W2"][e], w.act)
        ys[rows] += S_gpu[sample[rows], e][:, None] * out
    assert_y_close(to_np(y.float())[sample], ys, "bf16")


def test_expert_choice_many_ties_across_slices():
    """Coarse integer inputs make many tokens share an affinity exactly, so
    the cut-off of most experts falls inside a run of equal keys that spans
    several of the selection's slices; the choice must still be the first
    ones in position order (checked teacher-forced, bit-exact)."""
    w = Workload("ties", T=2003, d=16, E=8, k=2, H=64, act="swiglu", dtype="bf16", cf=1.0,
                 seed=25)
    inp = make_inputs(w, "cpu")
    g = torch.Generator().manual_seed(5)
    # every token is one of 12 distinct rows, so each expert's column holds
    # at most 12 distinct affinities
    rows = torch.randint(-1, 2, (12, w.d), generator=g).to(torch.bfloat16)
    inp["x"] = rows[torch.randint(0, 12, (w.T,), generator=g)].contiguous()
    inp["Wg"] = torch.randint(-1, 2, (w.d, w.E), generator=g).to(torch.bfloat16)
    t, layer, y, st, v = _run(w, inp)
    S_gpu = to_np(v["scores"]).T.astype(np.float64)
    n = v["n"]
    assert all(len(np.unique(S_gpu[:, e])) <= 12 for e in range(w.E))
    sel, tokens = oracle.expert_choice_select(S_gpu, n)
    pos = to_np(v["pos"])
    assert np.array_equal(pos >= 0, sel)
    tok = to_np(v["tok"])
    for e in range(w.E):
        assert np.array_equal(tok[e], tokens[e])


def test_expert_choice_long_slices_read_keys_from_memory():
    """T = 40000 tokens: each of the selection's four slices per expert holds
    10000 keys, more than its threads keep in registers, so the passes read
    the keys from the affinity matrix instead; the selection must be the
    same (teacher-forced, bit-exact, with ties from coarse inputs)."""
    w = Workload("long", T=40000, d=16, E=8, k=2, H=64, act="swiglu", dtype="bf16", cf=1.0,
                 seed=26)
    inp = make_inputs(w, "cpu")
    g = torch.Generator().manual_seed(6)
    rows = torch.randint(-2, 3, (50, w.d), generator=g).to(torch.bfloat16)
    inp["x"] = rows[torch.randint(0, 50, (w.T,), generator=g)].contiguous()
    t, layer, y, st, v = _run(w, inp)
    assert st.device_error == 0
    S_gpu = to_np(v["scores"]).T.astype(np.float64)
    n = v["n"]
    sel, tokens = oracle.expert_choice_select(S_gpu, n)
    pos = to_np(v["pos"])
    assert np.array_equal(pos >= 0, sel)
    tok = to_np(v["tok"])
    for e in range(w.E):
        assert np.array_equal(tok[e], tokens[e])
