"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these checks re-types the oracle's own formulas: each compares the
oracle with a worked example from the pages, a closed form, an identity the
pages state, or a brute-force computation written here independently (subset
enumeration, a sequential capacity queue, triple loops, a per-token loop with
no permutation).  Each is chosen so that a plausible slip in the oracle (a
dropped term, a swapped W1/W3, softmax over all experts, floor instead of ceil,
dropping early tokens instead of late ones, renormalising after a drop, a
transposed operand) fails at least one of them.
"""

import itertools
import math
import os

import numpy as np
import pytest

import oracle
from oracle import moe_oracle as O

RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------- helpers
def _read_golden(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def brute_matmul(a, b):
    n, m = a.shape
    m2, p = b.shape
    assert m == m2
    out = np.zeros((n, p))
    for i in range(n):
        for j in range(p):
            s = 0.0
            for c in range(m):
                s += a[i, c] * b[c, j]
            out[i, j] = s
    return out


def brute_silu(z):
    # SiLU written through the logistic function sigma(z) = e^z / (1 + e^z).
    return np.array([v * (math.exp(v) / (1.0 + math.exp(v))) if v < 0
                     else v / (1.0 + math.exp(-v)) for v in z.ravel()]
                    ).reshape(z.shape)


def brute_gelu(z):
    # GELU(z) = z * Phi(z), Phi the standard normal CDF via math.erfc.
    return np.array([v * 0.5 * math.erfc(-v / math.sqrt(2.0))
                     for v in z.ravel()]).reshape(z.shape)


def brute_ffn(xr, W1, W3, W2, act):
    if act == "swiglu":
        h = brute_silu(brute_matmul(xr, W1)) * brute_matmul(xr, W3)
    else:
        h = brute_gelu(brute_matmul(xr, W1))
    return brute_matmul(h, W2)


def brute_topk(logit_row, k):
    """Max-sum k-subset; among equal sums the lexicographically smallest set
    of indices; slots ordered by (-logit, index)."""
    E = len(logit_row)
    best, best_key = None, None
    for sub in itertools.combinations(range(E), k):
        key = (-sum(logit_row[i] for i in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return sorted(best, key=lambda i: (-logit_row[i], i))


def brute_capacity_queue(idx, E, C):
    """Sequential simulation: tokens arrive in position order; an expert
    accepts while it has room."""
    T, k = idx.shape
    used = [0] * E
    kept = np.zeros((T, k), dtype=bool)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if C is None or used[e] < C:
                kept[t, j] = True
            used[e] += 1
    return kept, np.array(used)


def brute_layer(x, Wg, bias, W1, W3, W2, k, C, act):
    """Per-token evaluation of y_t = sum over kept selected experts of
    gate * E_e(x_t), straight from the definition (no permutation)."""
    T = x.shape[0]
    E = Wg.shape[1]
    logits = brute_matmul(x, Wg)
    if bias is not None:
        logits = logits + bias[None, :]
    idx = np.array([brute_topk(list(logits[t]), k) for t in range(T)])
    kept, _ = brute_capacity_queue(idx, E, C)
    y = np.zeros((T, W2.shape[2]))
    for t in range(T):
        sel = [logits[t, e] for e in idx[t]]
        m = max(sel)
        w = [math.exp(v - m) for v in sel]
        s = sum(w)
        for j, e in enumerate(idx[t]):
            if not kept[t, j]:
                continue
            out = brute_ffn(x[t:t + 1], W1[e], None if W3 is None else W3[e],
                            W2[e], act)[0]
            y[t] += (w[j] / s) * out
    return y, idx, kept


def rand_layer(T, d, E, H, act, bias=False, int_valued=False):
    if int_valued:
        x = RNG.integers(-3, 4, size=(T, d)).astype(float)
        Wg = RNG.integers(-2, 3, size=(d, E)).astype(float)
    else:
        x = RNG.standard_normal((T, d))
        Wg = RNG.standard_normal((d, E)) / math.sqrt(d)
    b = RNG.standard_normal(E) * 0.5 if bias else None
    W1 = RNG.standard_normal((E, d, H)) / math.sqrt(d)
    W3 = RNG.standard_normal((E, d, H)) / math.sqrt(d) if act == "swiglu" else None
    W2 = RNG.standard_normal((E, H, d)) / math.sqrt(H)
    return x, Wg, b, W1, W3, W2


# ----------------------------------------------------------------- gating
def test_golden_top2_gates_07_03(golden_dir):
    g = {r[0]: r[1:] for r in _read_golden(os.path.join(golden_dir, "gates_top2_07_03.txt"))}
    logits = np.array([[float(v) for v in g["logits"]]])
    k = int(g["k"][0])
    idx, sel, _ = O.top_k(logits, k)
    gate = O.gating_softmax(sel)
    assert idx[0].tolist() == [int(v) for v in g["idx"]]
    np.testing.assert_allclose(gate[0], [float(v) for v in g["gates"]],
                               rtol=0, atol=1e-15)


@pytest.mark.parametrize("E,k", [(4, 1), (8, 2), (32, 2), (64, 8), (8, 8)])
def test_selected_gates_sum_to_one(E, k):
    logits = RNG.standard_normal((200, E)) * 3
    _, sel, _ = O.top_k(logits, k)
    gate = O.gating_softmax(sel)
    np.testing.assert_allclose(gate.sum(1), 1.0, rtol=0, atol=1e-14)
    assert (gate > 0).all()
    # Softmax over *all* experts followed by TopK would not sum to one: the
    # pinned quantity really depends on the order TopK -> Softmax.
    if k < E:
        dense = np.exp(logits - logits.max(1, keepdims=True))
        dense /= dense.sum(1, keepdims=True)
        assert (np.sort(dense, 1)[:, -k:].sum(1) < 1 - 1e-6).all()


def test_top1_gate_is_one():
    logits = RNG.standard_normal((100, 6))
    _, sel, _ = O.top_k(logits, 1)
    assert np.all(O.gating_softmax(sel) == 1.0)


@pytest.mark.parametrize("E,k", [(4, 1), (5, 2), (6, 3), (8, 2), (8, 4)])
def test_topk_matches_subset_bruteforce(E, k):
    # Small-integer logits make ties frequent and sums exact.
    logits = RNG.integers(-2, 3, size=(300, E)).astype(float)
    idx, _, margin = O.top_k(logits, k)
    for t in range(logits.shape[0]):
        assert idx[t].tolist() == brute_topk(list(logits[t]), k)
        srt = sorted(logits[t], reverse=True)
        want = srt[k - 1] - srt[k] if k < E else math.inf
        assert margin[t] == want


def test_topk_tie_goes_to_lower_index():
    logits = np.array([[0.5, 2.0, 2.0, 1.0, 2.0]])
    idx, _, margin = O.top_k(logits, 2)
    assert idx[0].tolist() == [1, 2]
    assert margin[0] == 0.0


# --------------------------------------------------------------- capacity
def test_capacity_golden(golden_dir):
    for T, E, k, cf, C in _read_golden(os.path.join(golden_dir, "capacity_values.txt")):
        assert O.capacity(int(T), int(E), int(k), float(cf)) == int(C)


def test_dropless_capacity_values():
    assert O.capacity(100, 4, 2, 0.0) is None
    assert O.capacity(100, 4, 2, -1.0) is None
    assert O.capacity(100, 4, 2, math.inf) is None
    assert O.capacity(100, 4, 2, None) is None


@pytest.mark.parametrize("T,E,k,C", [(64, 4, 1, 10), (64, 4, 2, 20), (50, 8, 3, 5),
                                      (64, 4, 2, None), (33, 6, 2, 0), (40, 5, 5, 7)])
def test_capacity_matches_sequential_queue(T, E, k, C):
    logits = RNG.standard_normal((T, E))
    logits[:, 0] += 1.0  # skew load toward expert 0 so drops happen
    idx, _, _ = O.top_k(logits, k)
    counts, kept_counts, rank, kept = O.assign_capacity(idx, E, C)
    want_kept, want_counts = brute_capacity_queue(idx, E, C)
    assert (kept == want_kept).all()
    assert (counts == want_counts).all()
    assert (kept_counts == (want_counts if C is None else np.minimum(want_counts, C))).all()
    # rank = number of earlier tokens queued at the same expert
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            assert rank[t, j] == np.sum(idx[:t] == e)


def test_infinite_capacity_drops_nothing():
    x, Wg, b, W1, W3, W2 = rand_layer(64, 8, 4, 16, "swiglu")
    r = O.moe_forward(x, Wg, b, W1, W3, W2, 2, 0.0, "swiglu")
    assert r["C"] is None and r["kept"].all()
    assert (r["kept_counts"] == r["counts"]).all()
    assert r["counts"].sum() == 64 * 2


def test_drops_fall_on_the_latest_tokens():
    """Drop-towards-the-End: at every expert, each dropped assignment comes
    after every kept one in token position."""
    T, E, k = 400, 8, 2
    logits = RNG.standard_normal((T, E))
    logits[:, :2] += 1.5
    idx, _, _ = O.top_k(logits, k)
    C = O.capacity(T, E, k, 1.0)
    _, _, _, kept = O.assign_capacity(idx, E, C)
    assert not kept.all()
    for e in range(E):
        tk = np.nonzero((idx == e) & kept)[0]
        td = np.nonzero((idx == e) & ~kept)[0]
        if td.size and tk.size:
            assert td.min() > tk.max()


# ------------------------------------------------------------ activations
def test_activation_closed_forms():
    # Phi(1) = 0.8413447460685429..., Phi(-1) = 1 - Phi(1) (textbook values)
    np.testing.assert_allclose(O.gelu(np.array([1.0, -1.0, 0.0])),
                               [0.8413447460685429, -0.15865525393145707, 0.0],
                               rtol=1e-15, atol=1e-17)
    np.testing.assert_allclose(O.silu(np.array([0.0, math.log(3.0)])),
                               [0.0, math.log(3.0) * 0.75], rtol=1e-15)
    z = RNG.standard_normal(1000) * 4
    # odd-part identities: f(z) - f(-z) = z for both SiLU and GELU
    np.testing.assert_allclose(O.silu(z) - O.silu(-z), z, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(O.gelu(z) - O.gelu(-z), z, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(O.silu(z), brute_silu(z), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(O.gelu(z), brute_gelu(z), rtol=1e-14, atol=1e-15)
    # Large negative inputs: SiLU tends to 0 without producing NaN.
    assert O.silu(np.array([-1000.0]))[0] == 0.0


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_expert_ffn_matches_triple_loops(act):
    d, H = 12, 20
    xr = RNG.standard_normal((5, d))
    W1 = RNG.standard_normal((d, H)) / math.sqrt(d)
    W3 = RNG.standard_normal((d, H)) / math.sqrt(d)
    W2 = RNG.standard_normal((H, d)) / math.sqrt(H)
    got = O.expert_ffn(xr, W1, W3 if act == "swiglu" else None, W2, act)
    want = brute_ffn(xr, W1, W3 if act == "swiglu" else None, W2, act)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)
    if act == "swiglu":
        # SiLU sits on the W1 branch: swapping W1 and W3 changes the result.
        swapped = O.expert_ffn(xr, W3, W1, W2, act)
        assert np.abs(swapped - want).max() > 1e-3


# ---------------------------------------------------------- whole layer
def dense_ffn(x, W1, W3, W2, act):
    return brute_ffn(x, W1, W3, W2, act)


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_single_expert_reduces_to_dense_ffn(act):
    """E = 1, k = 1, infinite capacity: the layer is the dense FFN."""
    x, Wg, b, W1, W3, W2 = rand_layer(6, 8, 1, 16, act)
    r = O.moe_forward(x, Wg, b, W1, W3, W2, 1, 0.0, act)
    want = dense_ffn(x, W1[0], None if W3 is None else W3[0], W2[0], act)
    np.testing.assert_allclose(r["y"], want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("k", [1, 2, 4])
def test_upcycling_identity(k):
    """All experts copies of one FFN, TopK then Softmax, dropless: the MoE
    output equals the dense FFN ("[Paper Club] Upcycling ...": the upcycled
    model behaves exactly like the dense one before training)."""
    E, d, H = 6, 8, 16
    x, Wg, b, W1, W3, W2 = rand_layer(10, d, E, H, "swiglu", bias=True)
    W1[:] = W1[0]
    W3[:] = W3[0]
    W2[:] = W2[0]
    r = O.moe_forward(x, Wg, b, W1, W3, W2, k, 0.0, "swiglu")
    want = dense_ffn(x, W1[0], W3[0], W2[0], "swiglu")
    np.testing.assert_allclose(r["y"], want, rtol=1e-12, atol=1e-12)


def test_granularity_identity():
    """Fine-grained upcycling ("[Paper Club] Upcycling ...", fine-grained
    MoE): experts are the G shards (split along H) of copies of one FFN and
    the router columns are duplicated inside each copy, so TopG picks every
    shard of the best copy once, each gate is 1/G and y = FFN(x) / G.  The
    duplicated columns also make exact logit ties."""
    n_copies, G, d, H = 3, 4, 8, 32
    E = n_copies * G
    T = 12
    x = RNG.standard_normal((T, d))
    R = RNG.standard_normal((d, n_copies))
    Wg = np.repeat(R, G, axis=1)  # column c*G+s = R[:, c]
    W1f = RNG.standard_normal((d, H)) / math.sqrt(d)
    W3f = RNG.standard_normal((d, H)) / math.sqrt(d)
    W2f = RNG.standard_normal((H, d)) / math.sqrt(H)
    hs = H // G
    W1 = np.stack([W1f[:, s * hs:(s + 1) * hs] for c in range(n_copies) for s in range(G)])
    W3 = np.stack([W3f[:, s * hs:(s + 1) * hs] for c in range(n_copies) for s in range(G)])
    W2 = np.stack([W2f[s * hs:(s + 1) * hs, :] for c in range(n_copies) for s in range(G)])
    r = O.moe_forward(x, Wg, None, W1, W3, W2, G, 0.0, "swiglu")
    best = np.argmax(x @ R, axis=1)
    for t in range(T):
        assert sorted(r["idx"][t].tolist()) == list(range(best[t] * G, best[t] * G + G))
    np.testing.assert_allclose(r["gate"], 1.0 / G, rtol=0, atol=1e-15)
    want = dense_ffn(x, W1f, W3f, W2f, "swiglu") / G
    np.testing.assert_allclose(r["y"], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act,k,cf,bias,int_valued", [
    ("swiglu", 2, 0.0, False, False),
    ("swiglu", 2, 1.0, True, False),
    ("gelu", 1, 1.25, False, False),
    ("swiglu", 3, 0.75, False, True),   # integer-valued routing: many ties
])
def test_layer_matches_per_token_bruteforce(act, k, cf, bias, int_valued):
    T, d, E, H = 24, 6, 5, 10
    x, Wg, b, W1, W3, W2 = rand_layer(T, d, E, H, act, bias=bias, int_valued=int_valued)
    C = O.capacity(T, E, k, cf)
    r = O.moe_forward(x, Wg, b, W1, W3, W2, k, cf, act)
    y, idx, kept = brute_layer(x, Wg, b, W1, W3, W2, k, C, act)
    assert (r["idx"] == idx).all()
    assert (r["kept"] == kept).all()
    np.testing.assert_allclose(r["y"], y, rtol=1e-11, atol=1e-12)


def test_dropped_slot_is_not_renormalised():
    """A token whose second slot is dropped keeps gate g0 < 1 on its first
    expert: y = g0 * E_0(x), not E_0(x)."""
    T, d, E, H, k = 8, 4, 2, 6, 2
    x, Wg, b, W1, W3, W2 = rand_layer(T, d, E, H, "swiglu")
    r = O.moe_forward(x, Wg, b, W1, W3, W2, k, 0.5, "swiglu")  # C = 4
    assert r["C"] == 4
    # Every token picks both experts; tokens 4..7 are dropped at both.
    assert r["kept"][:4].all() and not r["kept"][4:].any()
    assert np.all(r["y"][4:] == 0.0)
    t = 0
    parts = [r["gate"][t, j] * O.expert_ffn(x[t:t + 1], W1[e], W3[e], W2[e], "swiglu")[0]
             for j, e in enumerate(r["idx"][t])]
    np.testing.assert_allclose(r["y"][t], parts[0] + parts[1], rtol=1e-12)


def test_token_subset_matches_full_layer():
    T, d, E, H, k = 30, 6, 6, 8, 2
    x, Wg, b, W1, W3, W2 = rand_layer(T, d, E, H, "swiglu", bias=True)
    r = O.moe_forward(x, Wg, b, W1, W3, W2, k, 1.0, "swiglu")
    rows = np.array([0, 5, 17, 29])
    y, gate = O.moe_forward_tokens(x[rows], r["logits"][rows], r["idx"][rows],
                                   r["kept"][rows], W1, W3, W2, "swiglu")
    np.testing.assert_allclose(y, r["y"][rows], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(gate, r["gate"][rows], rtol=1e-15)


# ------------------------------------------------ Switch-order gating
def test_golden_switch_order_gates_04_02(golden_dir):
    g = {r[0]: r[1:] for r in _read_golden(os.path.join(golden_dir, "gates_switch_order_04_02.txt"))}
    logits = np.array([[float(v) for v in g["logits"]]])
    k = int(g["k"][0])
    idx, sel, _ = O.top_k(logits, k)
    assert idx[0].tolist() == [int(v) for v in g["idx"]]
    gate = O.gating_softmax_all(logits, idx)
    np.testing.assert_allclose(gate[0], [float(v) for v in g["gates"]], rtol=0, atol=1e-15)
    E = logits.shape[1]
    r = O._gates(logits, idx, sel, "softmax_topk", E / k)
    np.testing.assert_allclose(r[0], [float(v) for v in g["scaled"]], rtol=0, atol=1e-15)


def test_switch_order_gates_are_the_dense_probabilities():
    """Softmax-then-TopK gates are the dense softmax probabilities of the
    selected experts: they sum to less than one unless k = E, and the
    selection is the same as TopK of the logits."""
    logits = RNG.standard_normal((300, 8)) * 2
    idx, sel, _ = O.top_k(logits, 2)
    g = O.gating_softmax_all(logits, idx)
    dense = np.exp(logits) / np.exp(logits).sum(1, keepdims=True)
    for t in range(300):
        order = sorted(range(8), key=lambda e: (-dense[t, e], e))[:2]
        assert idx[t].tolist() == order
        np.testing.assert_allclose(g[t], dense[t, idx[t]], rtol=1e-13)
    assert (g.sum(1) < 1).all()
    idx8, sel8, _ = O.top_k(logits, 8)
    np.testing.assert_allclose(O.gating_softmax_all(logits, idx8).sum(1), 1.0, atol=1e-14)


def test_switch_order_upcycling_scale_restores_dense_output():
    """Identical experts and a uniform router (all logits equal): every
    softmax probability is 1/E, top-k gates sum to k/E, and the E/k scale of
    "[Paper Club] Upcycling ..." brings the output back to the dense FFN."""
    E, k, d, H = 8, 2, 8, 16
    x, Wg, b, W1, W3, W2 = rand_layer(10, d, E, H, "swiglu")
    Wg[:] = 0.0
    W1[:] = W1[0]
    W3[:] = W3[0]
    W2[:] = W2[0]
    dense = dense_ffn(x, W1[0], W3[0], W2[0], "swiglu")
    r = O.moe_forward(x, Wg, None, W1, W3, W2, k, 0.0, "swiglu", gating="softmax_topk",
                      gate_scale=E / k)
    np.testing.assert_allclose(r["gate"], 0.5, atol=1e-15)
    np.testing.assert_allclose(r["y"], dense, rtol=1e-12, atol=1e-12)
    r1 = O.moe_forward(x, Wg, None, W1, W3, W2, k, 0.0, "swiglu", gating="softmax_topk")
    np.testing.assert_allclose(r1["y"], dense * k / E, rtol=1e-12, atol=1e-12)


# ------------------------------------------------ Batch Priority Routing
def brute_priority_queue(idx, prio, E, C):
    """Sequential simulation: tokens arrive in descending priority (ties by
    position); an expert accepts while it has room."""
    T, k = idx.shape
    arrival = sorted(range(T), key=lambda t: (-prio[t], t))
    used = [0] * E
    kept = np.zeros((T, k), dtype=bool)
    for t in arrival:
        for j in range(k):
            e = int(idx[t, j])
            if used[e] < C:
                kept[t, j] = True
            used[e] += 1
    return kept


@pytest.mark.parametrize("T,E,k,cf", [(64, 4, 1, 0.5), (80, 8, 2, 1.0), (50, 6, 3, 0.6)])
def test_priority_capacity_matches_sequential_queue(T, E, k, cf):
    logits = RNG.standard_normal((T, E)) * 2
    logits[:, 0] += 1.0
    idx, sel, _ = O.top_k(logits, k)
    gate = O.gating_softmax(sel)
    # quantised gates make exact priority ties frequent
    gate = np.round(gate * 8) / 8 + 1e-9 * (gate == 0)
    C = O.capacity(T, E, k, cf)
    _, kept_counts, _, kept = O.assign_capacity(idx, E, C, O.priority_order(gate))
    assert (kept == brute_priority_queue(idx, gate[:, 0], E, C)).all()
    assert (kept_counts == np.minimum(np.bincount(idx.ravel(), minlength=E), C)).all()


def test_priority_drops_least_important_tokens():
    """At every expert, each dropped assignment has a priority no higher than
    every kept one ("Priority Routing": the least important are skipped)."""
    T, E, k = 300, 8, 2
    logits = RNG.standard_normal((T, E))
    logits[:, :2] += 1.5
    idx, sel, _ = O.top_k(logits, k)
    gate = O.gating_softmax(sel)
    C = O.capacity(T, E, k, 1.0)
    _, _, _, kept = O.assign_capacity(idx, E, C, O.priority_order(gate))
    assert not kept.all()
    for e in range(E):
        pk = gate[:, 0][np.nonzero((idx == e) & kept)[0]]
        pd = gate[:, 0][np.nonzero((idx == e) & ~kept)[0]]
        if pk.size and pd.size:
            assert pd.max() <= pk.min()


@pytest.mark.parametrize("T,E,k,cf,bounds", [
    (200, 8, 2, 1.0, (0, 70, 130, 200)),
    (96, 4, 1, 0.5, (0, 0, 50, 96)),       # an empty shard
    (150, 6, 3, 0.8, (0, 1, 149, 150)),    # one-token shards
    (64, 8, 2, 0.0, (0, 32, 64)),          # dropless
])
def test_sharded_capacity_concatenates_to_whole_batch(T, E, k, cf, bounds):
    """Shards of a batch, each given the assignments of the lower-position
    shards, keep exactly the assignments the whole batch keeps: checked
    against the one-at-a-time queue on the whole batch."""
    logits = RNG.standard_normal((T, E))
    logits[:, 0] += 1.2  # a hot expert, so capacity binds
    idx, _, _ = O.top_k(logits, k)
    C = O.capacity(T, E, k, cf)
    want = brute_capacity_queue(idx, E, C)[0]
    prior = np.zeros(E, dtype=np.int64)
    got = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        counts, kept_counts, _, kept = O.assign_capacity_shard(idx[a:b], E, C, prior)
        assert (kept_counts == kept.reshape(-1).astype(np.int64) @ np.eye(E, dtype=np.int64)[
            idx[a:b].reshape(-1)]).all()
        got.append(kept)
        prior = prior + np.bincount(idx[a:b].reshape(-1), minlength=E)
    assert (np.concatenate(got) == want).all()


# ------------------------------------------------ expert-choice routing
def test_golden_expert_choice_t5_e2(golden_dir):
    g = {r[0]: r[1:] for r in _read_golden(os.path.join(golden_dir, "expert_choice_t5_e2.txt"))}
    logits = np.array([[float(v) for v in g[f"logits_{t}"]] for t in range(5)])
    k = int(g["k"][0])
    S = O.expert_choice_scores(logits)
    np.testing.assert_allclose(S[:, 0], [0.75, 0.5, 0.25, 0.9, 0.5], rtol=0, atol=1e-15)
    for case in ("case_a", "case_b"):
        cf, C = float(g[case][0]), int(g[case][1])
        assert O.capacity(5, 2, k, cf) == C
        sel, tokens = O.expert_choice_select(S, C)
        assert tokens[0].tolist() == [int(v) for v in g[case + "_e0"]]
        assert tokens[1].tolist() == [int(v) for v in g[case + "_e1"]]
        np.testing.assert_allclose((S * sel).sum(1), [float(v) for v in g[case + "_weight"]],
                                   rtol=0, atol=1e-15)


def brute_expert_choice(scores, C):
    """Selection by the defining property, with loops only: expert e takes
    min(C, T) tokens, and every taken token beats every other token (larger
    score, or an equal score at a lower position)."""
    T, E = scores.shape
    n = min(C, T)
    sel = np.zeros((T, E), dtype=bool)
    for e in range(E):
        for t in range(T):
            # tokens that beat t at expert e
            better = 0
            for u in range(T):
                if scores[u, e] > scores[t, e] or (scores[u, e] == scores[t, e] and u < t):
                    better += 1
            sel[t, e] = better < n
    return sel


@pytest.mark.parametrize("T,E,C", [(12, 3, 4), (9, 4, 9), (10, 2, 15), (7, 5, 0), (16, 4, 5)])
def test_expert_choice_selection_matches_definition(T, E, C):
    # quantised scores make exact ties common
    scores = np.round(RNG.random((T, E)) * 4) / 4
    sel, tokens = O.expert_choice_select(scores, C)
    assert (sel == brute_expert_choice(scores, C)).all()
    assert (sel.sum(0) == min(C, T)).all()
    for e in range(E):
        assert tokens[e].tolist() == sorted(tokens[e].tolist())


def test_expert_choice_uniform_router_takes_the_first_tokens():
    """W_g = 0: every affinity is 1/E, so every expert takes tokens 0..C-1;
    with identical experts y_t = FFN(x_t) there (sum of E weights 1/E) and
    0 for the tokens no expert took."""
    T, d, E, H, k, cf = 20, 6, 4, 10, 1, 1.0
    x = RNG.standard_normal((T, d))
    W1 = np.repeat(RNG.standard_normal((1, d, H)), E, 0)
    W3 = np.repeat(RNG.standard_normal((1, d, H)), E, 0)
    W2 = np.repeat(RNG.standard_normal((1, H, d)), E, 0)
    r = O.moe_forward_expert_choice(x, np.zeros((d, E)), None, W1, W3, W2, k, cf, "swiglu")
    C = r["C"]
    assert C == 5
    assert all(t.tolist() == list(range(C)) for t in r["tokens"])
    dense = brute_ffn(x, W1[0], W3[0], W2[0], "swiglu")
    np.testing.assert_allclose(r["y"][:C], dense[:C], rtol=1e-12, atol=1e-12)
    assert (r["y"][C:] == 0).all()


def test_expert_choice_single_expert_is_dense():
    T, d, H = 9, 5, 7
    x = RNG.standard_normal((T, d))
    W1, W3, W2 = (RNG.standard_normal((1, d, H)), RNG.standard_normal((1, d, H)),
                  RNG.standard_normal((1, H, d)))
    r = O.moe_forward_expert_choice(x, RNG.standard_normal((d, 1)), None, W1, W3, W2, 1, 1.0,
                                    "swiglu")
    np.testing.assert_allclose(r["y"], brute_ffn(x, W1[0], W3[0], W2[0], "swiglu"),
                               rtol=1e-12, atol=1e-12)


def test_expert_choice_with_room_for_every_token_is_token_choice_top_e():
    """C >= T: every expert takes every token, y = sum_e softmax_e * E_e(x),
    which is the dropless token-choice layer with k = E."""
    T, d, E, H = 11, 6, 3, 8
    x, Wg, bias, W1, W3, W2 = rand_layer(T, d, E, H, "swiglu", bias=True)
    r = O.moe_forward_expert_choice(x, Wg, bias, W1, W3, W2, E, 1.0, "swiglu")
    assert r["C"] >= T and r["sel"].all()
    ref = O.moe_forward(x, Wg, bias, W1, W3, W2, E, 0.0, "swiglu")
    np.testing.assert_allclose(r["y"], ref["y"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act", ["swiglu", "gelu"])
def test_expert_choice_layer_matches_per_token_bruteforce(act):
    T, d, E, H, k, cf = 14, 5, 4, 6, 2, 0.75
    x, Wg, bias, W1, W3, W2 = rand_layer(T, d, E, H, act, bias=True)
    r = O.moe_forward_expert_choice(x, Wg, bias, W1, W3, W2, k, cf, act)
    logits = brute_matmul(x, Wg) + bias[None, :]
    y = np.zeros((T, d))
    C = math.ceil(cf * T * k / E)
    S = np.zeros((T, E))
    for t in range(T):
        m = max(logits[t])
        w = [math.exp(v - m) for v in logits[t]]
        S[t] = [v / sum(w) for v in w]
    sel = brute_expert_choice(S, C)
    for t in range(T):
        for e in range(E):
            if sel[t, e]:
                y[t] += S[t, e] * brute_ffn(x[t:t + 1], W1[e], None if W3 is None else W3[e],
                                            W2[e], act)[0]
    assert (r["sel"] == sel).all()
    np.testing.assert_allclose(r["y"], y, rtol=1e-10, atol=1e-12)
