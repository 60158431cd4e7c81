"""Failure detection on the GPU, without faulting it.

* A bad offsets table (a block that does not start on a 128-row boundary,
  one that runs past the buffer) is turned by the grouped GEMM's own checks
  into an error bit; the other experts are still computed.
* A wait that runs out: the MMA issuer of one up projection is made to wait
  on a barrier nobody arms (MOE_DEBUG_STALL_MMA, read once per process, so
  the test runs in a child process).  Every role gives up within its bounded
  wait (2 s), the forward reports MOE_ERR_DEVICE with the time-out bits, and
  the next forward in the same process is correct: the context survives.
"""

import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_51_b200 import moe as M

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ERR_TIMEOUT_MMA = 1 << 1
ERR_ROW_OVERFLOW = 1 << 4


def test_bad_offsets_are_reported_and_skipped():
    torch.manual_seed(1)
    E, d, H = 4, 128, 256
    kept = [100, 100, 100, 50]
    off = [0, 64, 256, 1024, 1152]  # expert 1 misaligned, expert 3 past the rows
    rows = 384
    xp = torch.randn(rows, d).bfloat16()
    W1 = (torch.randn(E, d, H) / d ** 0.5).bfloat16()
    W3 = (torch.randn(E, d, H) / d ** 0.5).bfloat16()
    W2 = (torch.randn(E, H, d) / H ** 0.5).bfloat16()
    dev = torch.device("cuda")
    offs = torch.tensor(off, dtype=torch.int32, device=dev)
    kc = torch.tensor(kept, dtype=torch.int32, device=dev)
    h = torch.zeros(rows, H, dtype=torch.bfloat16, device=dev)
    o = torch.zeros(rows, d, dtype=torch.bfloat16, device=dev)
    h, o, err = M.moe_grouped_ffn(xp.to(dev), offs, kc, W1.to(dev), W3.to(dev), W2.to(dev),
                                  "swiglu", h=h, o=o)
    torch.cuda.synchronize()
    assert int(err.item()) & ERR_ROW_OVERFLOW
    o = o.float().cpu().numpy()
    h = h.float().cpu().numpy()
    for e in (0, 2):  # the well-formed experts are still computed
        r = slice(off[e], off[e] + kept[e])
        xr = xp[r].double().numpy()
        h_ref = oracle.silu(xr @ W1[e].double().numpy()) * (xr @ W3[e].double().numpy())
        assert np.all(np.abs(h[r] - h_ref) <= 2.0 ** -8 * np.abs(h_ref) + 1e-6)
        o_ref = h[r].astype(np.float64) @ W2[e].double().numpy()
        # o is rounded to bf16 once
        assert np.all(np.abs(o[r] - o_ref) <= 2.0 ** -8 * np.abs(o_ref) + 1e-4)
    # nothing was written for the skipped experts' rows that no block owns
    assert np.all(o[128:256] == 0)


CHILD = textwrap.dedent("""
    import sys, torch
    sys.path.insert(0, {root!r})
    from mixture_experts_layer_51_b200 import moe as M
    from mixture_experts_layer_51_b200.workloads import Workload, make_inputs
    w = Workload("stall", T=600, d=256, E=8, k=2, H=384, act="swiglu", dtype="bf16",
                 cf=0.0, seed=13)
    t = make_inputs(w, "cuda")
    layer = M.MoELayer(t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act)
    try:
        layer(t["x"], stats=True)
        print("NO_ERROR")
    except M.MoeError as exc:
        assert exc.status == M.MOE_ERR_DEVICE, exc
        err = int(layer.intermediates(w.T)["dev_error"].item())
        print("DEVICE_ERROR", err)
    y1, st1 = layer(t["x"], stats=True)
    y2, st2 = layer(t["x"], stats=True)
    torch.cuda.synchronize()
    assert st1.device_error == 0 and st2.device_error == 0
    assert torch.isfinite(y1.float()).all() and torch.equal(y1, y2)
    print("RECOVERED")
""")


def test_stalled_wait_times_out_and_the_context_survives():
    env = dict(os.environ, MOE_DEBUG_STALL_MMA="1")
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = r.stdout.split("\n")
    err_line = [ln for ln in lines if ln.startswith("DEVICE_ERROR")]
    assert err_line, r.stdout
    assert int(err_line[0].split()[1]) & ERR_TIMEOUT_MMA
    assert "RECOVERED" in lines


CANARY = 0xA5


@pytest.mark.parametrize("case", [
    dict(T=1000, d=256, E=8, k=2, H=384, cf=0.0),
    dict(T=1100, d=136, E=6, k=3, H=200, cf=0.5),
    dict(T=700, d=256, E=64, k=8, H=384, cf=1.25),
])
def test_no_writes_outside_the_caller_buffers(case):
    """Every output and the workspace are bracketed by canary bytes; a
    forward (token choice, then expert choice) must leave them untouched."""
    from mixture_experts_layer_51_b200.workloads import Workload, make_inputs
    w = Workload("canary", act="swiglu", dtype="bf16", seed=17, **case)
    t = make_inputs(w, "cuda")
    pad = 4096

    def bracketed(nbytes):
        buf = torch.full((nbytes + 2 * pad,), CANARY, dtype=torch.uint8, device="cuda")
        return buf, buf[pad:pad + nbytes]

    def intact(buf, nbytes):
        head, tail = buf[:pad], buf[pad + nbytes:]
        return bool((head == CANARY).all()) and bool((tail == CANARY).all())

    need = M.moe_workspace_bytes(w.T, w.d, w.H, w.E, w.k, w.cf, torch.bfloat16, w.act)
    ws_buf, ws = bracketed(need)
    ybytes = w.T * w.d * 2
    y_buf, y_raw = bracketed(ybytes)
    y = y_raw.view(torch.bfloat16).view(w.T, w.d)
    M.moe_forward(t["x"], t["Wg"], t["bias"], t["W1"], t["W3"], t["W2"], w.k, w.cf, w.act, y=y,
                  ws=ws)
    torch.cuda.synchronize()
    assert intact(ws_buf, need) and intact(y_buf, ybytes)
    assert torch.isfinite(y.float()).all()

    ec_cf = w.cf if w.cf > 0 else 1.0
    L = M.moe_expert_choice_layout(w.T, w.d, w.H, w.E, w.k, ec_cf, "bf16", w.act)
    ws_buf, ws = bracketed(L.total)
    y_buf, y_raw = bracketed(ybytes)
    y = y_raw.view(torch.bfloat16).view(w.T, w.d)
    st = M.lib().moe_forward_expert_choice(
        M._ptr(t["x"]), M._ptr(t["Wg"]), M._ptr(t["bias"]), M._ptr(t["W1"]), M._ptr(t["W3"]),
        M._ptr(t["W2"]), w.T, w.d, w.H, w.E, w.k, ec_cf, M.MOE_SWIGLU, M.MOE_BF16, M._ptr(y),
        M._ptr(ws), ws.numel(), None, M._stream(y.device))
    assert st == M.MOE_OK
    torch.cuda.synchronize()
    assert intact(ws_buf, L.total) and intact(y_buf, ybytes)

