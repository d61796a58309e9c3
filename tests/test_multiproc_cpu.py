"""The multi-rank plumbing of bench.py, exercised as two gloo ranks on CPU:
max-over-ranks timing, the barrier, whole-job throughput of independent
replicas (each rank its own seeded inputs, no data-path exchange), and the
reference arm that only rank 0 runs."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank times its own replica; the job time is the slowest rank's
        my_ms = 10.0 + 5.0 * rank
        ms = bench.dist_max(my_ms)
        bench.dist_barrier()
        value = bench.job_throughput(units_per_rank=100, world=world, max_ms=ms)
        # the reference arm runs on rank 0 only; other ranks return at once
        class A:
            steps, warmup, tokens = 1, 0, 1
        ref = bench.run_reference(A(), lambda m: None) if rank != 0 else "skipped on rank 0"
        q.put((rank, ms, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_job_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, value, ref in res:
        assert ms == 15.0  # max over ranks, seen identically by every rank
        assert value == pytest.approx(100 * 2 / 0.015)
    assert res[1][3] is None  # rank 1 does no reference work


def test_replica_seeds_differ_per_rank():
    """Each replica draws its own inputs (seed 1000 + rank in the decode leg)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    x0, l0 = bench.layer_inputs(1000, 0, 1)
    x1, l1 = bench.layer_inputs(1001, 0, 1)
    assert not np.array_equal(x0, x1) and not np.array_equal(l0, l1)
