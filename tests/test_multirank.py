"""The N > 1 path of bench.py, on CPU ranks over gloo (world size 2).

Each rank runs its own full replica of the workload (weak scaling, no
collective on the data path); the only collective is the timing reduction,
which must take the slowest rank's time and count every rank's units.  The
CPU-oracle reference arm runs on rank 0 only; other ranks exit at once.
"""
import io
import os
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms_local = 2.0 + rank            # rank 1 is the slower one
    ms_max, value = bench.aggregate_over_ranks(ms_local, amount=3.0, world=world,
                                               device=torch.device("cpu"))
    # the reference arm: rank 0 prints, the others return without work
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.run_reference(bench.parse_args(["--impl", "reference", "--config", "issue-repro",
                                                   "--steps", "1", "--warmup", "0",
                                                   "--cpu-seconds", "0.1"])) if rank == 1 else 0
    results[rank] = (ms_max, value, rc, buf.getvalue())
    dist.barrier()
    dist.destroy_process_group()


def test_timing_reduction_takes_the_slowest_rank():
    world = 2
    port = 29500 + (os.getpid() % 1000)
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    for rank in range(world):
        ms_max, value, rc, out = res[rank]
        assert ms_max == 3.0
        assert abs(value - world * 3.0 / 3e-3) < 1e-6   # units of both ranks / slowest time
        assert rc == 0
    assert res[1][3] == ""                               # non-zero ranks print nothing


def test_single_rank_aggregation_is_local():
    import bench
    ms, value = bench.aggregate_over_ranks(4.0, amount=2.0, world=1, device=torch.device("cpu"))
    assert ms == 4.0 and abs(value - 500.0) < 1e-9
