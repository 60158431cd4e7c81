"""The routers other than the default streaming one, forced on: the
tensor-core router (route_tc.cu) and the clustered mma.sync router
(route.cu), on small batches, ragged sizes, both gate orders and expert
choice.  The choice (MOE_ROUTE_STREAM, MOE_ROUTE_TC) is read once per
process, so each check runs in a child."""

import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


ALTERNATES = {"tensor_core": {"MOE_ROUTE_STREAM": "0", "MOE_ROUTE_TC": "1"},
              "mma_sync_clusters": {"MOE_ROUTE_STREAM": "0", "MOE_ROUTE_TC": "0"}}


@pytest.mark.parametrize("router", list(ALTERNATES))
def test_alternate_router_forced_on_small_batches(router):
    """An alternate router forced on the small parity layers and a ragged
    batch must still match the oracle."""
    script = textwrap.dedent("""
        import sys
        sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
        from parity import full_parity
        from mixture_experts_layer_51_b200.workloads import WORKLOADS, Workload, make_inputs
        cases = [
            WORKLOADS["top2_bf16"].replace(T=600, d=256, H=384),
            WORKLOADS["mixtral_bf16"].replace(T=520, d=512, H=640),
            WORKLOADS["finegrained_bf16"].replace(T=700, d=256, H=384),
            WORKLOADS["openmoe_skew_bf16"].replace(T=1100, d=256, H=512, seq_len=275),
            Workload("ragged", T=333, d=200, E=16, k=4, H=256, act="swiglu", dtype="bf16",
                     cf=0.75, seed=27),
        ]
        for w in cases:
            full_parity(w, make_inputs(w, "cpu"))
            full_parity(w, make_inputs(w, "cpu"), gating="softmax_topk", gate_scale=2.0)
        print("TC_ROUTER_OK")
    """).format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    env = dict(os.environ, **ALTERNATES[router])
    r = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    assert "TC_ROUTER_OK" in r.stdout


@pytest.mark.parametrize("router", list(ALTERNATES))
def test_alternate_router_expert_choice_forced(router):
    script = textwrap.dedent("""
        import sys
        sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
        import test_gpu_expert_choice as T
        for name in ("top2_bf16", "mixtral_bf16", "finegrained_bf16", "one_token",
                     "room_for_all"):
            w = T.CASES[name]
            T._check(w, T.make_inputs(w, "cpu"))
        print("TC_EC_OK")
    """).format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    env = dict(os.environ, **ALTERNATES[router])
    r = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    assert "TC_EC_OK" in r.stdout
