#!/usr/bin/env python
"""Benchmark of the MoE layer forward on B200: tokens/s and TFLOPS.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle, timed

One step = one moe_forward (router GEMM + TopK/softmax, permutation, grouped
SwiGLU FFN, combine) over one batch of synthetic tokens already resident in
HBM.  With N > 1 (launched by torch.distributed.run) every rank runs an
independent replica of the layer on its own batch (the forward has no data
exchange when dropless), the timed region is bracketed by a barrier and a
device synchronise, and the time is the max over ranks.  Rank 0 prints one
JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "mixtral_bf16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (profiling runs on a smaller batch)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (profiling runs with fewer experts' weights)")
    ap.add_argument("--hidden", type=int, default=None,
                    help="override H (profiling the router/permute/combine kernels)")
    ap.add_argument("--capacity-factor", type=float, default=None,
                    help="override the workload's capacity factor")
    ap.add_argument("--routing", choices=["token_choice", "expert_choice"],
                    default="token_choice",
                    help="expert_choice: every expert takes its top-C tokens "
                         "(capacity factor 1.0 unless one is given)")
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of replaying the forward's CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-kernels", action="store_true",
                    help="skip the back-to-back timing of the HBM-bound kernels")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the timed loops of the other layer shapes")
    ap.add_argument("--cpu-sample", type=int, default=None,
                    help="tokens per oracle sample (default: sized to ~10-20 s)")
    return ap.parse_args(argv)


# ----------------------------------------------------------- accounting
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def algorithmic(w, n_kept, tokens_with_kept, routing="token_choice"):
    """FLOPs and HBM bytes of each stage for one forward (padding and dropped
    assignments are never counted)."""
    s = 2 if w.dtype == "bf16" else 4
    T, d, E, k, H = w.T, w.d, w.E, w.k, w.H
    c_up = 4 if w.act == "swiglu" else 2
    flop = {
        "route": 2.0 * T * d * E,
        "ffn_up": c_up * float(d) * H * n_kept,
        "ffn_down": 2.0 * d * H * n_kept,
    }
    n_w_up = (2 if w.act == "swiglu" else 1) * E * d * H
    byts = {
        # read x and W_g once; write idx, gate (T*k each) and margin
        "route": T * d * s + d * E * s + T * k * 8 + T * 4,
        # read idx twice, the rows of x that are kept somewhere, write kept rows and pos
        "permute": 2 * T * k * 4 + tokens_with_kept * d * s + n_kept * d * s + T * k * 4,
        # weights once, activations in and out
        "ffn_up": n_w_up * s + n_kept * d * s + n_kept * H * s,
        "ffn_down": E * H * d * s + n_kept * H * s + n_kept * d * s,
        # read kept rows of o (layer dtype), pos and gate; write y
        "combine": n_kept * d * s + T * k * 8 + T * d * s,
    }
    if routing == "expert_choice":
        # route: read x and W_g, write the [T, E] affinities; select + gather:
        # read the affinities, write pos [T, E] and the token lists, read each
        # chosen token's x row once and write one row per assignment; combine:
        # kept rows of o, pos and affinities [T, E], write y
        byts["route"] = T * d * s + d * E * s + T * E * 4
        byts["permute"] = 2 * T * E * 4 + n_kept * 4 + tokens_with_kept * d * s + n_kept * d * s
        byts["combine"] = n_kept * d * s + T * E * 8 + T * d * s
    total_flop = flop["route"] + flop["ffn_up"] + flop["ffn_down"]
    return flop, byts, total_flop


# A roofline fraction above this means the timed kernel is not doing the
# work it is credited with (or the wrong peak was used): the line is refused.
MAX_ROOFLINE_FRAC = 1.05


def choose_bf16_peak(peaks, loop_s, clk, src="measured"):
    """The bf16 denominator that fits the timed region, decided by the clocks
    sampled during it: the sustained (power-capped) figure when at least two
    samples show sw_power_cap and their median SM clock is below 92 % of max;
    the burst figure otherwise (full clock, a cap that only flickered, or no
    samples).  Returns (peak, description)."""
    sustained = (clk is not None and clk.get("samples", 0) >= 2
                 and "sw_power_cap" in clk.get("reasons", [])
                 and clk.get("sm_mhz", 0) < 0.92 * clk.get("sm_max_mhz", 1))
    clock = (f", median SM clock {clk['sm_mhz']:.0f} of {clk['sm_max_mhz']:.0f} MHz"
             f"{' (' + ', '.join(clk['reasons']) + ')' if clk.get('reasons') else ''}"
             if clk else ", clocks not sampled")
    if sustained:
        return peaks["bf16_tflops_sustained"], (
            f"{src} bf16 sustained: timed loop of {loop_s:.2f} s under the power cap{clock}")
    return peaks["bf16_tflops"], f"{src} bf16 burst: timed loop of {loop_s:.3f} s{clock}"


def roofline_fraction(achieved, peak):
    """achieved / peak, refusing a value no correct measurement can give."""
    if achieved is None or not peak:
        return None
    frac = achieved / peak
    if frac > MAX_ROOFLINE_FRAC:
        raise ValueError(f"roofline fraction {frac:.3f} > {MAX_ROOFLINE_FRAC}: "
                         f"{achieved:.1f} against a peak of {peak:.1f}")
    return round(frac, 4)


def traffic_for(kernel_file, kernel, w):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current source of the kernel and on this workload; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        src = os.path.join(ROOT, "mixture_experts_layer_51_b200", "csrc", kernel_file)
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if rec.get("source_sha") != sha:
            return None
        cfg = rec.get("config", {})
        if cfg != {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "H": w.H}:
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------- ranks
def rank_env():
    """(rank, local_rank, world) from the torch.distributed launcher env."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def max_over_ranks(value, device=None):
    """The largest of every rank's `value` (a time); identity on one rank.
    Every rank must call it at the same point (it is a collective)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, steps, elapsed_ms):
    """Units all ranks processed per second over the (max-over-ranks) time."""
    return world * units_per_rank * steps / (elapsed_ms / 1e3)


# --------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sms.append(float(r[1]))
                maxs.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "samples": len(sms), "reasons": sorted(reasons)}


# ---------------------------------------------------------- CPU oracle
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_seconds(w, cpu_inp, T_s, routing="token_choice"):
    """Run the fp64 oracle as it stands on the first T_s tokens (routing,
    capacity over that sample batch, expert FFNs, combine); wall seconds."""
    import oracle
    x = cpu_inp["x"][:T_s]
    t0 = time.perf_counter()
    if routing == "expert_choice":
        oracle.moe_forward_expert_choice(x, cpu_inp["Wg"], cpu_inp["bias"], cpu_inp["W1"],
                                         cpu_inp["W3"], cpu_inp["W2"], w.k, w.cf, w.act)
        return time.perf_counter() - t0
    logits = oracle.router_logits(x, cpu_inp["Wg"], cpu_inp["bias"])
    idx, _, _ = oracle.top_k(logits, w.k)
    C = oracle.capacity(T_s, w.E, w.k, w.cf)
    _, _, _, kept = oracle.assign_capacity(idx, w.E, C)
    oracle.moe_forward_tokens(x, logits, idx, kept, cpu_inp["W1"], cpu_inp["W3"],
                              cpu_inp["W2"], w.act)
    return time.perf_counter() - t0


def default_cpu_sample(w):
    # ~10-20 s of fp64 work on the host cores for the large layers
    # (measured: ~330 Mixtral-shaped tokens/s on 16 cores, ~230 GFLOP/s).
    per_token = 2.0 * w.k * (3 if w.act == "swiglu" else 2) * w.d * w.H
    return int(max(16, min(w.T, 3e12 / per_token)))


# ------------------------------------------------------------- timing
def forward_loop(step, steps, stream, dev, clocks=None, world=1):
    """K calls of step() between two events on the launching stream, bracketed
    by a barrier (N > 1) and a device synchronise; returns (ms, clocks)."""
    import torch
    import torch.distributed as dist
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if clocks:
        clocks.start()
        time.sleep(0.3)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop() if clocks else None
    return start.elapsed_time(end), clk


def stage_loop(M, layer, x, y, n, stream, dev):
    """n forwards with events recorded between the stages
    (moe_set_stage_events); returns the mean ms of each stage."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(M.MOE_NUM_STAGE_EVENTS)]
           for _ in range(n)]
    for row in evs:  # torch creates the CUDA event on first record
        for ev in row:
            ev.record(stream)
    torch.cuda.synchronize(dev)
    for i in range(n):
        M.moe_set_stage_events(evs[i])
        layer(x, y=y)
    M.moe_set_stage_events(None)
    torch.cuda.synchronize(dev)
    stage_ms = {s: 0.0 for s in M.STAGES}
    for i in range(n):
        for s, v in M.stage_times_ms(evs[i]).items():
            stage_ms[s] += v / n
    return stage_ms


def back_to_back_ms(launches, reps, stream, dev):
    """Mean ms per launch of `reps` rounds over the list `launches` (each a
    callable enqueuing one kernel on `stream`), launched back to back between
    two events after one untimed round."""
    import torch
    for fn in launches:
        fn()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(reps):
        for fn in launches:
            fn()
    end.record(stream)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end) / (reps * len(launches))


def hbm_kernels(M, w, layer, x, inp, byts, hbm, stream, dev):
    """The HBM-bound stages timed as kernels: each launched back to back
    through its own entry point on inputs that rotate through copies of x
    (more than twice the 126 MB L2 between two reads of one copy), beside a
    plain streaming read of the same bytes (moe_probe_stream_read).  The
    stage-event loop's figures include the gap every event opens between two
    kernels; these do not."""
    import torch
    T = w.T
    nbytes = x.numel() * x.element_size()
    copies = max(2, min(64, -(-252_000_000 // max(nbytes, 1)) + 1))
    xs = [x.clone() for _ in range(copies)]
    v = layer.intermediates(T)
    idx, gate, margin, pos = v["idx"], v["gate"], v["margin"], v["pos"]
    idx2, gate2, margin2 = torch.empty_like(idx), torch.empty_like(gate), torch.empty_like(margin)
    perm = {k: torch.empty_like(v[k]) for k in ("pos", "counts", "kept_counts", "offsets")}
    xp = torch.empty_like(v["xp"])
    ws = torch.empty(M.moe_permute_workspace_bytes(T, w.E), dtype=torch.uint8, device=dev)
    yb = torch.empty_like(x)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    reps = 10
    out = {}
    ms = back_to_back_ms([lambda xx=xx: M.moe_probe_stream_read(xx, sink) for xx in xs],
                         reps, stream, dev)
    out["plain_read"] = {"ms": round(ms, 5), "bytes": nbytes,
                         "gbs": round(nbytes / (ms / 1e3) / 1e9, 1),
                         "frac_hbm": round(nbytes / (ms / 1e3) / 1e9 / hbm, 4)}
    routes = [lambda xx=xx: M.moe_route(xx, inp["Wg"], inp["bias"], w.k, idx2, gate2, margin2)
              for xx in xs]
    permutes = [lambda xx=xx: M.moe_permute(xx, idx, w.E, w.cf, xp=xp, ws=ws, **perm)
                for xx in xs]
    combines = [lambda: M.moe_unpermute_combine(v["o"], pos, gate, x.dtype, y=yb)]
    for name, fns in (("route", routes), ("permute", permutes), ("combine", combines)):
        ms = back_to_back_ms(fns, reps if len(fns) > 1 else 2 * copies, stream, dev)
        gbs = byts[name] / (ms / 1e3) / 1e9
        out[name] = {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                     "of_plain_read": round(out["plain_read"]["ms"] * byts[name] / nbytes / ms, 4)}
    out["method"] = (f"before the timed loops (GPU at full clock), each entry point launched back "
                     f"to back ({reps} rounds over {copies} copies "
                     f"of x, {copies * nbytes / 1e6:.0f} MB; combine re-reads o "
                     f"{v['o'].numel() * v['o'].element_size() / 1e6:.0f} MB), CUDA events on "
                     "the launching stream; of_plain_read = the probe's time for the stage's "
                     "algorithmic bytes / the stage's time")
    del xs
    return out


def workload_record(M, w, make_inputs, peaks, peak_src, dev, stream, seconds=1.5,
                    sample_clocks=True):
    """One workload's forward, replayed as its CUDA graph in a timed loop of
    about `seconds` (clocks sampled), plus its stage breakdown."""
    import torch
    inp = make_inputs(w, dev)
    layer = M.MoELayer(inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], w.k, w.cf,
                       w.act, max_tokens=w.T)
    x = inp["x"]
    y = torch.empty_like(x)
    _, st = layer(x, y=y, stats=True)
    n_kept = int(st.kept)
    pos = layer.intermediates(w.T)["pos"]
    tokens_with_kept = int((pos >= 0).any(dim=1).sum().item())
    flop, byts, total_flop = algorithmic(w, n_kept, tokens_with_kept)
    graph = layer.graph(x, y)
    for _ in range(5):
        graph.launch()
    cal_ms, _ = forward_loop(graph.launch, 10, stream, dev)
    steps = int(min(50000, max(20, seconds * 1e3 / max(cal_ms / 10, 1e-3))))
    clocks = ClockSampler(dev.index or 0) if sample_clocks else None
    ms, clk = forward_loop(graph.launch, steps, stream, dev, clocks)
    graph.close()
    stage_ms = stage_loop(M, layer, x, y, 20, stream, dev)
    ms_step = ms / steps
    tflops = total_flop / (ms_step / 1e3) / 1e12
    rec = {"T": w.T, "d": w.d, "E": w.E, "k": w.k, "H": w.H, "act": w.act, "dtype": w.dtype,
           "capacity_factor": w.cf, "steps": steps, "ms_per_step": round(ms_step, 5),
           "tokens_per_s": round(w.T / (ms_step / 1e3), 1), "tflops": round(tflops, 2),
           "kept_assignments": n_kept, "clocks": clk,
           "stages_ms": {k: round(v, 5) for k, v in stage_ms.items()}}
    if w.dtype == "bf16":
        peak, src = choose_bf16_peak(peaks, ms / 1e3, clk, peak_src)
        rec.update({"frac_bf16_peak": roofline_fraction(tflops, peak), "peak": peak,
                    "peak_source": src})
    else:
        rec["bound"] = "latency (8.5 MFLOP per forward; a fraction of an FP32 peak means nothing)"
    del layer, inp, x, y
    torch.cuda.empty_cache()
    return rec


# ----------------------------------------------------------------- main
def main(argv=None):
    a = parse_args(argv)
    import torch
    import torch.distributed as dist

    from mixture_experts_layer_51_b200 import moe as M
    from mixture_experts_layer_51_b200.workloads import WORKLOADS, make_inputs

    rank, local, world = rank_env()
    w = WORKLOADS[a.workload]
    if a.tokens:
        w = w.replace(T=a.tokens)
    if a.experts:
        w = w.replace(E=a.experts)
    if a.hidden:
        w = w.replace(H=a.hidden)
    if a.capacity_factor is not None:
        w = w.replace(cf=a.capacity_factor)
    elif a.routing == "expert_choice" and not w.cf > 0:
        w = w.replace(cf=1.0)
    peaks, peak_src = load_peaks()

    if a.impl == "reference":
        return run_reference(a, w, rank, world)

    from datetime import timedelta
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    inp = make_inputs(w, dev)
    ec = a.routing == "expert_choice"
    if ec:
        layer = M.ExpertChoiceLayer(inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], w.k,
                                    w.cf, w.act)
    else:
        layer = M.MoELayer(inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], w.k, w.cf,
                           w.act, max_tokens=w.T)
    x = inp["x"]
    y = torch.empty_like(x)

    # Routing statistics for the FLOP count (kept assignments only).
    _, st = layer(x, y=y, stats=True)
    n_kept = int(st.kept)
    pos = layer.intermediates(w.T)["pos"]
    tokens_with_kept = int((pos >= 0).any(dim=1).sum().item())
    flop, byts, total_flop = algorithmic(w, n_kept, tokens_with_kept, a.routing)
    routing = None
    if not ec:
        try:
            routing = routing_report(w, list(st.counts), (pos >= 0).cpu().numpy())
        except Exception as exc:  # a report, never a reason to lose the measurement
            routing = {"error": str(exc)}

    # Token choice replays the forward as one CUDA graph (moe_forward_graph_*):
    # the same kernels, one host call per step, so layers whose forward is
    # shorter than the host's launch work are timed on the GPU, not the host.
    graph = None
    if not ec and not a.eager:
        try:
            graph = layer.graph(x, y)
        except M.MoeError as exc:
            print(f"graph capture unavailable ({exc}); timing eager launches", file=sys.stderr)
    launch_kind = "cuda_graph" if graph is not None else "eager"
    step = graph.launch if graph is not None else (lambda: layer(x, y=y))
    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize(dev)

    # The HBM-bound kernels timed alone, before the GEMM-heavy loops bring
    # the GPU to its power-capped clock (the stage loop below times them
    # inside the forward, in that regime).
    hbm = peaks["hbm_gbs"]
    kernels = None
    if not ec and world == 1 and not a.no_kernels:
        kernels = hbm_kernels(M, w, layer, x, inp, byts, hbm, stream, dev)

    # The timed loop: K forwards back to back, nothing recorded between
    # their kernels (an event between two kernels would stop the next one
    # from starting while the previous drains).
    clocks = ClockSampler(local) if not a.no_clocks else None
    elapsed_ms, clk = forward_loop(step, a.steps, stream, dev, clocks, world)
    if world > 1:
        dist.barrier()
    elapsed_ms = max_over_ranks(elapsed_ms, dev)

    # Stage breakdown from a separate loop with events recorded between the
    # stages (moe_set_stage_events), on the launching stream.
    n_stage = min(a.steps, 50)
    t_stage = time.perf_counter()
    stage_ms = stage_loop(M, layer, x, y, n_stage, stream, dev)
    stage_loop_s = time.perf_counter() - t_stage

    # Kernels of ours per timed forward: the kernel nodes of the captured
    # forward (token choice: router, placement + copy, two GEMMs, combine);
    # expert choice launches router, select, transpose, copy, two GEMMs and
    # combine.
    if ec:
        kernels_per_forward = 7
    else:
        try:
            g = graph if graph is not None else layer.graph(x, y=y)
            kernels_per_forward = g.nodes()[0]
            if g is not graph:
                g.close()
        except M.MoeError as exc:
            print(f"kernel count unavailable ({exc})", file=sys.stderr)
            kernels_per_forward = None
    ms_per_step = elapsed_ms / a.steps
    tokens_per_s = whole_job_rate(w.T, world, a.steps, elapsed_ms)
    tflops = total_flop * world * a.steps / (elapsed_ms / 1e3) / 1e12


    # End to end: every step copies its own batch from pinned host memory,
    # runs the layer and copies y back, through the streaming pipeline API
    # (four slots: the copies of some batches overlap the forward of another;
    # two already hide them on the Mixtral shape, the short forwards of the
    # small layers need more in flight).
    e2e = None
    if not a.no_e2e and not ec:
        depth = M.MOE_PIPELINE_MAX_DEPTH
        x_host = [x.cpu().pin_memory() for _ in range(depth)]
        y_host = [torch.empty_like(x_host[0]).pin_memory() for _ in range(depth)]
        pipe = M.Pipeline(layer, w.T, depth=depth)

        def stream_steps(n):
            for i in range(n):
                slot = i % depth
                if i >= depth:
                    pipe.wait(slot)
                pipe.submit(slot, x_host[slot], y_host[slot])
            for slot in range(min(n, depth)):
                pipe.wait(slot)

        stream_steps(2 * depth)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        stream_steps(a.steps)
        e1.record(stream)  # recorded after the host saw the last copy-out complete
        torch.cuda.synchronize(dev)
        pipe.close()
        e2e_ms = e0.elapsed_time(e1)
        e2e_ms = max_over_ranks(e2e_ms, dev)
        nbytes = x.numel() * x.element_size()
        e2e = {"value": whole_job_rate(w.T, world, a.steps, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "ms_per_step": e2e_ms / a.steps, "api": f"moe_pipeline_submit/wait, {depth} slots"}

    # CPU baseline: the oracle as it stands, bounded sample, rank 0 at N=1.
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu_inp = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in inp.items()}
        T_s = a.cpu_sample or default_cpu_sample(w)
        secs = oracle_sample_seconds(w, cpu_inp, T_s, a.routing)
        cpu = {"value": T_s / secs, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"first {T_s} tokens of the {w.name} batch (routing, capacity, expert "
                         f"FFNs, combine in fp64 NumPy), {secs:.1f} s"}
        del cpu_inp

    up_ms = stage_ms["ffn_up"]
    stages = {}
    for s in M.STAGES:
        ms = stage_ms[s]
        rec = {"ms": round(ms, 5)}
        if s in flop:
            rec["tflops"] = round(flop[s] / (ms / 1e3) / 1e12, 2) if ms > 0 else None
        rec["gbs"] = round(byts[s] / (ms / 1e3) / 1e9, 1) if ms > 0 else None
        if s in ("route", "permute", "combine") and rec["gbs"]:
            rec["frac_hbm"] = round(rec["gbs"] / hbm, 4)
        stages[s] = rec
    act_name = "SwiGLU" if w.act == "swiglu" else "GELU"
    achieved = flop["ffn_up"] / (up_ms / 1e3) / 1e12 if up_ms > 0 else None
    if w.dtype == "bf16":
        # The achieved rate comes from the stage loop, so its length and the
        # clocks of the headline loop just before it pick the peak.
        # (The stage loop follows the headline loop at once, so it runs in
        # the clock regime that loop's samples show.)
        roof_peak, roof_src = choose_bf16_peak(peaks, stage_loop_s, clk, peak_src)
        roofline = {"kernel": f"ffn_tc_kernel<{act_name}> (grouped up projection)",
                    "bound": "tensor",
                    "traffic": traffic_for("ffn_tc.cu", "ffn_up", w),
                    "peak_source": roof_src + f"; achieved from the stage loop of {n_stage} "
                                              "forwards"}
    else:
        # fp32 FMA on the SIMT pipes: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz
        roof_peak = FP32_SIMT_TFLOPS
        roofline = {"kernel": f"ffn_simt_kernel<{act_name}> (grouped up projection)",
                    "bound": "alu", "traffic": None,
                    "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz"}
    roofline.update({"achieved": round(achieved, 2) if achieved else None, "peak": roof_peak,
                     "unit": "TFLOP/s", "frac": roofline_fraction(achieved, roof_peak)})
    layer_peak, layer_src = (choose_bf16_peak(peaks, elapsed_ms / 1e3, clk, peak_src)
                             if w.dtype == "bf16" else (peaks["bf16_tflops"], ""))

    # The other layer shapes, each in a timed loop of its own (N = 1 only).
    others = None
    if rank == 0 and world == 1 and not a.no_workloads and not ec and a.workload == DEFAULT_WORKLOAD \
            and not (a.tokens or a.experts or a.hidden) and a.capacity_factor is None:
        if graph is not None:
            graph.close()
            graph = None
        del layer, inp, x, y
        torch.cuda.empty_cache()
        others = {}
        for name, wl in WORKLOADS.items():
            if name == w.name:
                continue
            try:
                others[name] = workload_record(M, wl, make_inputs, peaks, peak_src, dev, stream,
                                               sample_clocks=not a.no_clocks)
            except Exception as exc:  # one shape failing must not lose the headline
                others[name] = {"error": f"{type(exc).__name__}: {exc}"}

    if rank == 0:
        line = {
            "metric": "MoE layer fwd tokens/s (and TFLOPS as a fraction of bf16 dense peak) on 1 B200",
            "value": round(tokens_per_s, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded; random-init weights)",
            "config": {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "H": w.H,
                       "act": w.act, "capacity_factor": w.cf, "routing": a.routing,
                       "parallelism": f"replicas x{world}",
                       "launch": launch_kind,
                       "l2": l2_note(w)},
            "tflops": round(tflops, 2),
            "frac_bf16_peak": round(tflops / layer_peak, 4),
            "frac_bf16_peak_source": layer_src,
            "frac_bf16_peak_burst": round(tflops / peaks["bf16_tflops"], 4),
            "frac_bf16_peak_sustained": round(tflops / peaks["bf16_tflops_sustained"], 4),
            "kept_assignments": n_kept, "flop_per_step": total_flop, "routing_stats": routing,
            "stages": stages, "hbm_kernels": kernels, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": kernels_per_forward * a.steps if kernels_per_forward else None, "clocks": clk,
            "peaks": {**peaks, "source": peak_src},
            "workloads": others,
        }
        print(json.dumps(line), flush=True)
    if graph is not None:
        graph.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def routing_report(w, counts, kept_mask):
    """Observability of one forward's routing: load imbalance (largest
    expert count over the mean), assignments dropped by the capacity, and,
    with a capacity, the drop rate per octile of batch position and of
    position inside each sequence ("Drop-towards-the-End").  counts: [E]
    assignments per expert; kept_mask: [T, k] bool (pos >= 0)."""
    counts = np.asarray(counts[:w.E], dtype=np.float64)
    kept_mask = np.asarray(kept_mask, dtype=bool)
    rep = {"load_imbalance": round(float(counts.max() / max(counts.mean(), 1e-30)), 4),
           "assignments": int(kept_mask.size), "dropped": int((~kept_mask).sum())}
    if w.cf > 0 and w.T >= 8:
        seq = w.seq_len or w.T
        for label, p, span in (("drop_rate_by_batch_octile", np.arange(w.T), w.T),
                               ("drop_rate_by_sequence_octile", np.arange(w.T) % seq, seq)):
            step = max(1, span // 8)
            rep[label] = [round(float((~kept_mask[(p >= a) & (p < a + step)]).mean()), 4)
                          for a in range(0, step * 8, step) if ((p >= a) & (p < a + step)).any()]
    return rep


def l2_note(w):
    """Whether a step's inputs exceed the 126 MB L2 (no flush is done)."""
    s = 2 if w.dtype == "bf16" else 4
    wbytes = (3 if w.act == "swiglu" else 2) * w.E * w.d * w.H * s
    if wbytes + w.T * w.d * s > 126e6:
        return f"inputs larger than L2 (expert weights {wbytes / 1e9:.2f} GB stream from HBM every step)"
    return (f"inputs fit in L2 ({(wbytes + w.T * w.d * s) / 1e6:.1f} MB): no flush between "
            "steps; a latency-bound layer")


def run_reference(a, w, rank, world):
    """The oracle as it stands, on the host cores, on bounded samples of the
    same workload (rank 0 only)."""
    if rank != 0:
        return 0
    import torch
    from mixture_experts_layer_51_b200.workloads import make_inputs
    inp = make_inputs(w, "cuda" if torch.cuda.is_available() else "cpu")
    cpu_inp = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in inp.items()}
    del inp
    T_s = a.cpu_sample or max(8, default_cpu_sample(w) // 4)
    for _ in range(a.warmup):
        oracle_sample_seconds(w, cpu_inp, T_s)
    secs = [oracle_sample_seconds(w, cpu_inp, T_s) for _ in range(a.steps)]
    total = sum(secs)
    value = T_s * a.steps / total
    cores = cpu_threads()
    line = {
        "metric": "MoE layer fwd tokens/s (and TFLOPS as a fraction of bf16 dense peak) on 1 B200",
        "impl": "reference", "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(total / a.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; random-init weights)",
        "config": {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "H": w.H,
                   "act": w.act, "capacity_factor": w.cf},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"each step: first {T_s} tokens of the {w.name} batch"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
