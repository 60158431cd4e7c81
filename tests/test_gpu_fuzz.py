"""Randomised layer shapes against the fp64 oracle: 48 layers drawn from a
fixed seed -- both dtypes, 1 to 64 experts, top-1 to top-8, d and H from 8
to 512, 1 to 3000 tokens, dropless or with a capacity, SwiGLU or GELU, with
and without a router bias, both gate orders -- each checked whole (routing
away from near-ties, the permutation and every kept xp row bit-exact, every
element of y within the dtype's bound).  The shapes land on every router
back end, ragged tiles and tails the hand-picked cases may miss."""

import random

import pytest

from mixture_experts_layer_51_b200.workloads import Workload, make_inputs

from parity import full_parity

pytestmark = pytest.mark.gpu


def _draw(n, seed=2024):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        E = rng.choice([1, 2, 3, 4, 5, 6, 8, 12, 16, 24, 32, 40, 48, 64])
        k = rng.randint(1, min(E, 8))
        out.append(dict(
            name=f"fuzz{i}",
            T=rng.choice([1, 7, 64, 129, 300, 777, 1500, 3000]),
            d=8 * rng.randint(1, 64), H=8 * rng.randint(1, 64), E=E, k=k,
            act=rng.choice(["swiglu", "gelu"]),
            dtype=rng.choice(["bf16", "bf16", "fp32"]),
            cf=rng.choice([0.0, 0.0, 0.5, 1.0, 1.25]),
            seed=1000 + i,
            bias_var=rng.choice([0.0, 0.0, 0.5]),
            gating=rng.choice(["topk_softmax", "topk_softmax", "softmax_topk"])))
    return out


CASES = _draw(48)


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_random_layer_shape(case):
    case = dict(case)
    gating = case.pop("gating")
    w = Workload(**case)
    full_parity(w, make_inputs(w, "cpu"), gating=gating)
