"""fp64 NumPy oracle of one token-choice MoE FFN layer, forward pass.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this module and nothing here is shared with it.

Every array is cast to float64 on entry.  Inputs stored as bf16 are exactly
representable in float64, so the oracle sees the same numbers the GPU sees and
computes the definition without any intermediate rounding.

Readings of points the pages leave open:

* Order of TopK and Softmax: Softmax over the k selected logits (the Mixtral
  form in "The Math Behind MoEs"); the non-selected gates are 0.
* Ties in TopK: larger logit first; equal logits -> lower expert index first.
  The slot order j = 0..k-1 is that descending order.
* Router bias (when given): added to the logits before TopK and kept in the
  softmax.
* Capacity: C = ceil(cf * T * k / E) over the whole batch, evaluated in
  float64; cf <= 0 or inf means dropless.  Within an expert, assignments are
  served in ascending token position and the first C are kept ("Drop-towards-
  the-End").  A token never picks the same expert twice, so position alone
  orders an expert's queue.
* A dropped slot contributes 0 and the kept slots keep their gates (no
  renormalisation).
* SwiGLU expert: (SiLU(x W1) * (x W3)) W2, SiLU(z) = z / (1 + e^-z).
  GELU expert: GELU(x W1) W2 with the exact erf form.  No expert biases.
* Expert-choice routing ("[Paper Club] Upcycling ...", the Q&A on expert
  choice: the selection is reversed, every expert takes a fixed number of
  tokens, a token may get no expert, several, or all): the token-to-expert
  affinity is the router probability Softmax(x W_g) over all E experts (the
  G(x) of "The Math Behind MoEs" before any TopK); each expert takes the
  C = ceil(cf * T * k / E) tokens (at most T) with the largest affinity to it,
  equal affinities -> lower position first, k read as the average number of
  experts per token; the output is the affinity-weighted sum over the experts
  that took the token, with no renormalisation.
"""

from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

__all__ = [
    "router_logits",
    "top_k",
    "gating_softmax",
    "gating_softmax_all",
    "capacity",
    "assign_capacity",
    "priority_order",
    "silu",
    "gelu",
    "expert_ffn",
    "moe_forward",
    "moe_forward_tokens",
    "assign_capacity_shard",
    "expert_choice_scores",
    "expert_choice_select",
    "moe_forward_expert_choice",
]


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor (any dtype, CPU)
        a = a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


def router_logits(x, Wg, bias=None):
    """logits[t, e] = sum_c x[t, c] W_g[c, e] (+ bias[e]).

    "How do Mixture of Expert Models Work?", "The Math Behind MoEs": the gate
    acts on x . W_g; "[Paper Club] Upcycling ...": the router is a learnable
    matrix applied to the tokens.
    """
    logits = _f64(x) @ _f64(Wg)
    if bias is not None:
        logits = logits + _f64(bias)[None, :]
    return logits


def top_k(logits, k):
    """TopK of each row: indices (slot order = descending logit, ties -> lower
    index), the selected logits, and margin = k-th largest - (k+1)-th largest
    (+inf when k == E).

    "The Math Behind MoEs": Softmax(TopK(x . W_g)) keeps the k largest values.
    """
    logits = _f64(logits)
    T, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    # A stable sort of the negated logits puts equal logits in ascending
    # expert order, which is the tie rule.
    order = np.argsort(-logits, axis=1, kind="stable")
    idx = order[:, :k]
    sel = np.take_along_axis(logits, idx, axis=1)
    if k < E:
        nxt = np.take_along_axis(logits, order[:, k:k + 1], axis=1)[:, 0]
        margin = sel[:, k - 1] - nxt
    else:
        margin = np.full(T, np.inf)
    return idx.astype(np.int64), sel, margin


def gating_softmax(sel_logits):
    """Softmax over the k selected logits of each token (largest subtracted).

    "The Math Behind MoEs": the gating output is the softmax of only the top
    K values; "[Paper Club] Upcycling ...": with TopK before Softmax the
    selected gates always sum to one.
    """
    s = _f64(sel_logits)
    z = np.exp(s - s.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def gating_softmax_all(logits, idx):
    """Switch order, Softmax then TopK: the softmax over all E logits of each
    token, read at the selected experts.  The k gates no longer sum to one.

    "[Paper Club] Upcycling ...": the original Switch Transformer applies the
    softmax first, so the selected probabilities do not add up to one
    (example 0.4 and 0.2); "How do Mixture of Expert Models Work?", "The Math
    Behind MoEs": G(x) = Softmax(x . W_g).  TopK of the probabilities selects
    the same experts as TopK of the logits (softmax is increasing).
    """
    logits = _f64(logits)
    z = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = z / z.sum(axis=1, keepdims=True)
    return np.take_along_axis(p, np.asarray(idx, dtype=np.int64), axis=1)


def capacity(T, E, k, cf):
    """Per-expert capacity C = ceil(cf * T * k / E), or None when dropless.

    "How do Mixture of Expert Models Work?", "Expert Capacity": a cap on how
    many tokens one expert can see, typically a factor of 1 to 1.25;
    "[Paper Club] Upcycling ...": each expert accepts at most C tokens and
    the rest are dropped.  cf <= 0, None or inf means dropless.
    """
    if cf is None:
        return None
    cf = float(cf)
    if not math.isfinite(cf) or cf <= 0.0:
        return None
    return int(math.ceil(cf * T * k / E))


def priority_order(gate):
    """Batch Priority Routing order: tokens by descending importance, ties in
    ascending position.

    "Scaling Vision with Sparse Mixture of Experts", "Priority Routing":
    tokens are sorted by an importance score and the least important are the
    ones skipped when an expert is full.  The page does not define the score;
    it is read here as the token's largest gate (slot 0).
    """
    g = _f64(gate)
    return np.argsort(-g[:, 0], kind="stable")


def assign_capacity(idx, E, C, order=None):
    """Queue every (token, slot) assignment at its expert and keep the first
    C of each queue.  Tokens arrive in ascending position, or in `order` (a
    permutation of the tokens, e.g. priority_order) when given.

    Returns counts[E] (assignments per expert), kept_counts[E]
    (= min(count, C)), rank[T, k] (0-based place in the expert's queue) and
    kept[T, k] (bool).  "Take a Closer Look at the MoE LLM Routing",
    "Drop-towards-the-End": with position order, later tokens are the ones
    dropped.
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    if order is not None:
        order = np.asarray(order, dtype=np.int64)
        counts, kept_counts, rank_o, kept_o = assign_capacity(idx[order], E, C)
        rank = np.empty_like(rank_o)
        kept = np.empty_like(kept_o)
        rank[order] = rank_o
        kept[order] = kept_o
        return counts, kept_counts, rank, kept
    flat = idx.reshape(-1)  # token-major: (t, j) -> t * k + j
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    # Stable sort by expert keeps ascending token order inside each expert.
    order = np.argsort(flat, kind="stable")
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank_sorted = np.arange(flat.size) - np.repeat(starts, counts)
    rank = np.empty(flat.size, dtype=np.int64)
    rank[order] = rank_sorted
    rank = rank.reshape(T, k)
    if C is None:
        kept = np.ones((T, k), dtype=bool)
        kept_counts = counts.copy()
    else:
        kept = rank < C
        kept_counts = np.minimum(counts, C)
    return counts, kept_counts, rank, kept


def assign_capacity_shard(idx_shard, E, C, prior):
    """The capacity step for one shard of a batch whose tokens are split by
    position over ranks (shard r holds a contiguous range of positions).

    prior[e] counts the assignments to expert e from all lower-position
    shards.  In the whole batch's position-ordered queue of expert e, this
    shard's i-th assignment sits at place prior[e] + i, so it is kept iff
    that place is below C ("Drop-towards-the-End" applied to the whole
    batch, "Take a Closer Look at the MoE LLM Routing").  Returns counts,
    kept_counts, rank (local place) and kept as assign_capacity does.
    """
    counts, _, rank, _ = assign_capacity(idx_shard, E, None)
    idx_shard = np.asarray(idx_shard, dtype=np.int64)
    prior = np.asarray(prior, dtype=np.int64)
    if C is None:
        return counts, counts.copy(), rank, np.ones(rank.shape, dtype=bool)
    room = np.maximum(0, C - prior)
    kept = rank < room[idx_shard]
    return counts, np.minimum(counts, room), rank, kept


def silu(z):
    """SiLU(z) = z / (1 + exp(-z)) (the gate of SwiGLU)."""
    z = _f64(z)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def gelu(z):
    """Exact GELU(z) = z * Phi(z) = 0.5 z (1 + erf(z / sqrt 2))."""
    z = _f64(z)
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


def expert_ffn(xr, W1, W3, W2, act):
    """One expert's FFN on rows xr.

    act == "swiglu": (SiLU(xr W1) * (xr W3)) W2  (Mixtral's SwiGLU expert in
    "The Math Behind MoEs").  act == "gelu": GELU(xr W1) W2 (the original
    two-linear-layer FFN, "[Paper Club] Upcycling ...").
    """
    xr = _f64(xr)
    if act == "swiglu":
        h = silu(xr @ _f64(W1)) * (xr @ _f64(W3))
    elif act == "gelu":
        h = gelu(xr @ _f64(W1))
    else:
        raise ValueError(act)
    return h @ _f64(W2)


def _gates(logits, idx, sel, gating, gate_scale):
    if gating == "topk_softmax":
        gate = gating_softmax(sel)
    elif gating == "softmax_topk":
        gate = gating_softmax_all(logits, idx)
    else:
        raise ValueError(gating)
    return gate * float(gate_scale)


def _route(x, Wg, bias, k, gating="topk_softmax", gate_scale=1.0):
    logits = router_logits(x, Wg, bias)
    idx, sel, margin = top_k(logits, k)
    gate = _gates(logits, idx, sel, gating, gate_scale)
    return logits, idx, gate, margin


def moe_forward(x, Wg, bias, W1, W3, W2, k, cf, act, gating="topk_softmax", gate_scale=1.0,
                priority="position"):
    """The whole layer: route -> TopK + softmax -> capacity -> permute ->
    expert FFN -> un-permute with the gate-weighted sum.

    Returns a dict with y[T, d] and every intermediate: logits, idx, gate,
    margin, C, counts, kept_counts, rank, kept.  Steps follow the MoE-layer
    walk-through on "[Paper Club] Upcycling ..." and the formula
    y = sum_i G(x)_i E_i(x) of "The Math Behind MoEs".

    gating: "topk_softmax" (default, Mixtral) or "softmax_topk" (Switch
    order); gate_scale multiplies every gate ("[Paper Club] Upcycling ...":
    scaling the expert output by E/k restores the dense output scale when the
    softmax comes first, x4 for 8 experts and top-2).  priority: "position"
    (default; drop the latest tokens) or "gate" (Batch Priority Routing: drop
    the tokens with the smallest largest-gate first).
    """
    x = _f64(x)
    T, d = x.shape
    E = _f64(Wg).shape[1]
    logits, idx, gate, margin = _route(x, Wg, bias, k, gating, gate_scale)
    C = capacity(T, E, k, cf)
    order = priority_order(gate) if priority == "gate" else None
    counts, kept_counts, rank, kept = assign_capacity(idx, E, C, order)
    W1 = _f64(W1)
    W3 = _f64(W3) if W3 is not None else None
    W2 = _f64(W2)
    y = np.zeros((T, W2.shape[2]), dtype=np.float64)
    for e in range(E):
        # Permute: this expert's kept tokens in ascending position.
        tt, jj = np.nonzero((idx == e) & kept)
        if tt.size == 0:
            continue
        out = expert_ffn(x[tt], W1[e], None if W3 is None else W3[e], W2[e], act)
        # Un-permute, scaled by the router probability, summed over slots.
        y[tt] += gate[tt, jj][:, None] * out
    return dict(y=y, logits=logits, idx=idx, gate=gate, margin=margin, C=C,
                counts=counts, kept_counts=kept_counts, rank=rank, kept=kept)


def moe_forward_tokens(x_rows, logits_rows, sel_idx, kept, W1, W3, W2, act,
                       gating="topk_softmax", gate_scale=1.0):
    """The layer output for a subset of tokens, given their routing.

    x_rows[n, d], logits_rows[n, E] (the oracle's own fp64 logits),
    sel_idx[n, k] (the selected experts, slot order) and kept[n, k].  Gates
    are the softmax of the oracle's logits over the selected experts.  This
    lets a test check sampled tokens of a large batch, and check a batch whose
    selection at a near-tied logit differs, without running every token.
    """
    x_rows = _f64(x_rows)
    logits_rows = _f64(logits_rows)
    sel_idx = np.asarray(sel_idx, dtype=np.int64)
    kept = np.asarray(kept, dtype=bool)
    gate = _gates(logits_rows, sel_idx, np.take_along_axis(logits_rows, sel_idx, axis=1),
                  gating, gate_scale)
    n = sel_idx.shape[0]
    # W1/W3/W2 may be full [E, ...] arrays or dicts {expert: matrix}; only the
    # experts that are used get converted to float64.
    d_out = _f64(W2[int(sel_idx.flat[0])]).shape[1]
    y = np.zeros((n, d_out), dtype=np.float64)
    for e in np.unique(sel_idx):
        rr, jj = np.nonzero((sel_idx == e) & kept)
        if rr.size == 0:
            continue
        out = expert_ffn(x_rows[rr], W1[e], None if W3 is None else W3[e],
                         W2[e], act)
        y[rr] += gate[rr, jj][:, None] * out
    return y, gate


def expert_choice_scores(logits):
    """Token-to-expert affinity for expert-choice routing: the softmax of
    each token's logits over all E experts (largest subtracted)."""
    logits = _f64(logits)
    z = np.exp(logits - logits.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def expert_choice_select(scores, C):
    """Each expert's choice: sel[t, e] is True iff token t is among the
    min(C, T) tokens with the largest scores[:, e], equal scores taken in
    ascending position.  Returns sel [T, E] (bool) and, per expert, its
    chosen tokens in ascending position (the order of its rows)."""
    scores = _f64(scores)
    T, E = scores.shape
    n = min(int(C), T)
    sel = np.zeros((T, E), dtype=bool)
    for e in range(E):
        # stable sort of the negated scores: descending score, ties by position
        order = np.argsort(-scores[:, e], kind="stable")
        sel[order[:n], e] = True
    tokens = [np.nonzero(sel[:, e])[0] for e in range(E)]
    return sel, tokens


def moe_forward_expert_choice(x, Wg, bias, W1, W3, W2, k, cf, act, scores=None):
    """The layer with expert-choice routing: affinity -> every expert takes
    its top-C tokens -> expert FFN on them -> each token sums
    affinity * output over the experts that took it (ascending expert).

    cf must be > 0 (the experts' fixed intake is C = ceil(cf * T * k / E)).
    scores: optional [T, E] affinities to select on instead of the oracle's
    own (to replay another implementation's fp32 decision); the outputs are
    then weighted by those given scores too.
    """
    x = _f64(x)
    T = x.shape[0]
    E = _f64(Wg).shape[1]
    C = capacity(T, E, k, cf)
    if C is None:
        raise ValueError("expert-choice routing needs a finite capacity factor")
    logits = router_logits(x, Wg, bias)
    S = expert_choice_scores(logits) if scores is None else _f64(scores)
    sel, tokens = expert_choice_select(S, C)
    W2 = _f64(W2)
    y = np.zeros((T, W2.shape[2]), dtype=np.float64)
    for e in range(E):
        tt = tokens[e]
        if tt.size == 0:
            continue
        out = expert_ffn(x[tt], _f64(W1[e]), None if W3 is None else _f64(W3[e]), W2[e], act)
        y[tt] += S[tt, e][:, None] * out
    return dict(y=y, logits=logits, scores=S, C=C, sel=sel, tokens=tokens)
