"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws random numbers and names shapes.  It holds none of the
layer's arithmetic (no routing, capacity, activation or combine), so both the
CUDA path's tests and the CPU oracle's tests can take their inputs from here.

Workloads (sizes and distributions of the five layer shapes the MoE pages
discuss: a Switch-style tiny layer, a top-2 SwiGLU layer, the Mixtral 8x7B
layer shape, an OpenMoE-style skewed layer and a fine-grained layer):

* x ~ N(0, 1) unless ``tokens == "zipf"``.
* Router W_g [d, E] ~ N(0, 1/d); expert W1, W3 [E, d, H] ~ N(0, 1/d);
  W2 [E, H, d] ~ N(0, 1/H)  (variance = 1/fan_in).
* ``tokens == "zipf"``: token ids drawn (inverse CDF) from P(r) ~ r^-1.1 over
  a 32000-id vocabulary; x = emb[id] + 0.1 N(0, 1) with emb ~ N(0, 1) [32000, d], so the
  routing is dominated by the token id ("Context-independent Specialization"
  on "Take a Closer Look at the MoE LLM Routing").
* ``bias_var > 0``: a per-expert router bias ~ N(0, bias_var) in fp32.

Everything is drawn in fp32 from one ``torch.Generator`` seeded with the
workload's seed, in the fixed order x, W_g, bias, W1, W3, W2, and then cast to
the workload's storage dtype.  The same seed on a different device gives a
different (but again fixed) stream, so one run draws its inputs once and hands
the same tensors to both sides.
"""

from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    H: int
    act: str          # "swiglu" | "gelu"
    dtype: str        # "bf16" | "fp32"
    cf: float         # capacity factor; <= 0 means dropless
    seed: int
    tokens: str = "normal"   # "normal" | "zipf"
    bias_var: float = 0.0
    seq_len: int = 0         # sequence length for position reporting (0 = T)

    def replace(self, **kw):
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


WORKLOADS = {
    w.name: w
    for w in [
        Workload("switch_tiny_fp32", T=256, d=64, E=4, k=1, H=128, act="gelu",
                 dtype="fp32", cf=1.25, seed=0),
        Workload("top2_bf16", T=4096, d=1024, E=8, k=2, H=3584, act="swiglu",
                 dtype="bf16", cf=0.0, seed=1),
        Workload("mixtral_bf16", T=8192, d=4096, E=8, k=2, H=14336,
                 act="swiglu", dtype="bf16", cf=0.0, seed=2),
        Workload("openmoe_skew_bf16", T=16384, d=2048, E=32, k=2, H=8192,
                 act="swiglu", dtype="bf16", cf=1.0, seed=3, tokens="zipf",
                 seq_len=2048),
        Workload("finegrained_bf16", T=16384, d=2048, E=64, k=8, H=1408,
                 act="swiglu", dtype="bf16", cf=0.0, seed=4, bias_var=0.5),
    ]
}

ZIPF_VOCAB = 32000
ZIPF_S = 1.1


def _zipf_ids(gen, n, device):
    """n token ids with P(id = r - 1) proportional to r^-ZIPF_S, r = 1..ZIPF_VOCAB,
    by inverse-CDF sampling: one uniform draw per id and a binary search in
    the fp64 CDF (built on the host).  Unlike a multinomial draw on the GPU,
    this gives the same ids for the same seed in every process."""
    ranks = torch.arange(1, ZIPF_VOCAB + 1, dtype=torch.float64)
    cdf = torch.cumsum(ranks.pow(-ZIPF_S), 0)
    cdf = (cdf / cdf[-1]).to(device)
    u = torch.rand(n, generator=gen, device=device, dtype=torch.float64)
    return torch.searchsorted(cdf, u, right=True).clamp_(max=ZIPF_VOCAB - 1)


def _normal(gen, shape, std, device):
    return torch.randn(shape, generator=gen, device=device,
                       dtype=torch.float32) * std


def make_inputs(w: Workload, device="cpu"):
    """Draw the workload's inputs on ``device``.

    Returns a dict with x [T, d], Wg [d, E], bias [E] (fp32) or None,
    W1 [E, d, H], W3 [E, d, H] (None for GELU), W2 [E, H, d] and, for the
    Zipf workload, the token ids [T] (int64).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = w.torch_dtype
    out = {}
    if w.tokens == "zipf":
        ids = _zipf_ids(gen, w.T, device)
        emb = _normal(gen, (ZIPF_VOCAB, w.d), 1.0, device)
        x = emb[ids] + _normal(gen, (w.T, w.d), 0.1, device)
        del emb
        out["ids"] = ids
    else:
        x = _normal(gen, (w.T, w.d), 1.0, device)
    out["x"] = x.to(dt).contiguous()
    out["Wg"] = _normal(gen, (w.d, w.E), 1.0 / math.sqrt(w.d), device).to(dt)
    if w.bias_var > 0:
        out["bias"] = _normal(gen, (w.E,), math.sqrt(w.bias_var), device)
    else:
        out["bias"] = None
    out["W1"] = _normal(gen, (w.E, w.d, w.H), 1.0 / math.sqrt(w.d),
                        device).to(dt)
    if w.act == "swiglu":
        out["W3"] = _normal(gen, (w.E, w.d, w.H), 1.0 / math.sqrt(w.d),
                            device).to(dt)
    else:
        out["W3"] = None
    out["W2"] = _normal(gen, (w.E, w.H, w.d), 1.0 / math.sqrt(w.H),
                        device).to(dt)
    return out


def small_variant(w: Workload, T=None, d=None, H=None, E=None, k=None):
    """The same workload family at reduced sizes (for parity runs the oracle
    finishes in seconds)."""
    kw = {}
    for key, val in (("T", T), ("d", d), ("H", H), ("E", E), ("k", k)):
        if val is not None:
            kw[key] = val
    return w.replace(name=w.name + "_small", **kw)
