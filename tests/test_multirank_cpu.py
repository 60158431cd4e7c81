"""The N > 1 path of bench.py on CPU: two gloo ranks.

Every rank runs an independent replica on its own batch; the timed region is
reduced with a max over ranks and the whole-job rate counts every rank's
tokens.  The reference arm runs on rank 0 only; other ranks exit cleanly.
"""

import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, local, w = bench.rank_env()
        # rank r "took" 10 + r ms: every rank must see the slowest one
        t = bench.max_over_ranks(10.0 + r)
        rate = bench.whole_job_rate(units_per_rank=8192, world=w, steps=5, elapsed_ms=t)
        results[rank] = (r, w, t, rate)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        r, w, t, rate = results[rank]
        assert (r, w) == (rank, world)
        assert t == 11.0                       # the slowest rank's time
        assert rate == pytest.approx(2 * 8192 * 5 / 0.011)


def test_single_rank_helpers_without_process_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_rate(100, 1, 10, 1000.0) == pytest.approx(1000.0)


def test_reference_arm_nonzero_rank_exits_cleanly():
    """Under torchrun every rank runs `bench.py --impl reference`; only rank 0
    does work, the others exit 0 at once."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def _shard_worker(rank, world, port, bounds, results):
    """One rank of a position-sharded batch: its counts go through the
    package's all-gather; the capacity rule is the oracle's."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np

    import oracle
    from mixture_experts_layer_51_b200.sharded import gather_expert_counts
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, E, k, cf = 240, 8, 2, 1.0
        rng = np.random.default_rng(7)
        logits = rng.standard_normal((T, E))
        logits[:, 1] += 1.3
        idx, _, _ = oracle.top_k(logits, k)
        a, b = bounds[rank], bounds[rank + 1]
        counts = torch.as_tensor(np.bincount(idx[a:b].reshape(-1), minlength=E), dtype=torch.int32)
        gathered = gather_expert_counts(counts)
        prior = gathered[:rank].sum(0).numpy()
        _, _, _, kept = oracle.assign_capacity_shard(idx[a:b], E, oracle.capacity(T, E, k, cf),
                                                     prior)
        results[rank] = (gathered.numpy().tolist(), kept.tolist())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_sharded_capacity_exchange_gloo():
    """Two ranks holding positions [0, 100) and [100, 240) of one batch keep,
    after exchanging per-expert counts, exactly what the whole batch keeps."""
    import numpy as np

    import oracle
    world, bounds = 2, (0, 100, 240)
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, port, bounds, results), nprocs=world,
                       join=True, start_method="spawn")
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((240, 8))
    logits[:, 1] += 1.3
    idx, _, _ = oracle.top_k(logits, 2)
    _, _, _, want = oracle.assign_capacity(idx, 8, oracle.capacity(240, 8, 2, 1.0))
    assert not want.all()  # capacity binds, so the exchange matters
    g0, kept0 = results[0]
    g1, kept1 = results[1]
    assert g0 == g1 == [np.bincount(idx[a:b].reshape(-1), minlength=8).tolist()
                        for a, b in zip(bounds[:-1], bounds[1:])]
    assert (np.concatenate([np.array(kept0), np.array(kept1)]) == want).all()


def test_bench_algorithmic_units_and_l2_note():
    """The roofline's algorithmic units: FLOPs and bytes of each stage, kept
    assignments only, o counted in the layer dtype."""
    import bench
    from mixture_experts_layer_51_b200.workloads import WORKLOADS
    w = WORKLOADS["mixtral_bf16"]
    T, d, E, k, H = w.T, w.d, w.E, w.k, w.H
    n_kept = T * k
    flop, byts, total = bench.algorithmic(w, n_kept, T)
    assert flop["ffn_up"] == 4 * d * H * n_kept and flop["ffn_down"] == 2 * d * H * n_kept
    assert total == 2 * T * d * E + 6 * d * H * n_kept
    assert byts["route"] == T * d * 2 + d * E * 2 + 8 * T * k + 4 * T
    assert byts["combine"] == n_kept * d * 2 + 8 * T * k + T * d * 2
    assert byts["ffn_down"] == E * H * d * 2 + n_kept * H * 2 + n_kept * d * 2
    f32 = WORKLOADS["switch_tiny_fp32"]
    _, b32, _ = bench.algorithmic(f32, 200, 200)
    assert b32["combine"] == 200 * f32.d * 4 + 8 * f32.T * f32.k + f32.T * f32.d * 4
    assert bench.l2_note(w).startswith("inputs larger than L2")
    assert bench.l2_note(f32).startswith("inputs fit in L2")


def test_bench_routing_report():
    """Load imbalance, drops and drop rate by position octile from counts and
    the kept mask (the statistics forward's numbers)."""
    import numpy as np
    import bench
    from mixture_experts_layer_51_b200.workloads import WORKLOADS
    w = WORKLOADS["openmoe_skew_bf16"].replace(T=64, E=4, k=2, seq_len=16, cf=1.0)
    kept = np.ones((64, 2), dtype=bool)
    kept[48:, 1] = False            # the last quarter of the batch loses its 2nd slot
    counts = [64, 32, 16, 16]
    r = bench.routing_report(w, counts, kept)
    assert r["load_imbalance"] == 2.0 and r["assignments"] == 128 and r["dropped"] == 16
    assert r["drop_rate_by_batch_octile"] == [0, 0, 0, 0, 0, 0, 0.5, 0.5]
    # position inside each 16-token sequence: only the last sequence drops
    assert r["drop_rate_by_sequence_octile"] == [0.125] * 8
    dropless = bench.routing_report(w.replace(cf=0.0), counts, np.ones((64, 2), bool))
    assert dropless["dropped"] == 0 and "drop_rate_by_batch_octile" not in dropless
