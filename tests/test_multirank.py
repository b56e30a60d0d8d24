"""The multi-GPU path's host logic on CPU ranks (gloo, world size 2).

Heads and batches are independent, so ranks run disjoint seeded batches with
no collective on the data path (weak scaling); the only exchange is the MAX of
the per-rank device times, and the job's throughput is every rank's work over
that slowest time.  These are bench.py's helpers, run as two spawned processes.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    from exact_io_aware_100_b200 import inputs
    w = inputs.WORKLOADS["prefill"]
    seed = bench.rank_seed(w, rank)
    x = inputs.make_tensor(seed, "q", (2, 3, 16, 8))
    gathered = [torch.zeros(x.size, dtype=torch.int32) for _ in range(world)]
    dist.all_gather(gathered, torch.from_numpy(x.astype(np.int32).ravel()))
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, world, "cpu")
    dist.barrier()
    dist.destroy_process_group()
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), seed=seed, ms=ms,
             distinct=not torch.equal(gathered[0], gathered[1]))


def test_two_ranks_take_disjoint_batches_and_the_slowest_time(tmp_path):
    world, port = 2, _free_port()
    mp.spawn(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    r = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    assert int(r[0]["seed"]) != int(r[1]["seed"])
    assert bool(r[0]["distinct"]) and bool(r[1]["distinct"])
    assert float(r[0]["ms"]) == float(r[1]["ms"]) == 15.0


def test_job_throughput_counts_every_rank():
    import bench
    assert bench.job_tflops(2e12, 1, 10, 20.0) == pytest.approx(1000.0)
    assert bench.job_tflops(2e12, 4, 10, 20.0) == pytest.approx(4000.0)
    assert bench.max_over_ranks(3.5, None, 1, "cpu") == 3.5
