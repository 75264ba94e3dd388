"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): per-rank seeds give
distinct batches of the same shape, the job time is the slowest rank's, and the job value
sums every rank's work."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from datetime import timedelta

    import numpy as np
    import torch.distributed as dist

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    w = bench.rank_workload(synth.workloads()["fp8_8b"], rank)
    k = synth.keys(w, 0, 1, 0, 1, 0, 4)
    t = bench.max_over_ranks(1.0 + rank, world)  # rank 1 is slower
    v = bench.job_value(100e9, 10, t, world)
    out[rank] = (w.seed, float(np.abs(k.astype(np.float64)).sum()), t, v)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_plumbing():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork of a process that already runs threads
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    s0, k0, t0, v0 = out[0]
    s1, k1, t1, v1 = out[1]
    assert s0 != s1 and k0 != k1                 # distinct batches per rank
    assert t0 == t1 == 2.0                       # every rank reports the slowest interval
    assert v0 == v1 == pytest.approx(2 * 100 * 10 / 2.0)  # whole-job GB/s over both ranks
