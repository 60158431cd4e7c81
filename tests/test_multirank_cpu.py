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
