"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): each rank gets its own
independent batch of the same workload (weak scaling, no collective on the data path), the job's
time is the maximum over ranks and its units are the sum over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads as W
        cfg = W.CONFIGS["tiny"]
        w = W.make_workload(cfg, seed=cfg.seed + 1000 * rank)
        # Each rank times its own batch; the job takes the slowest rank and sums the units.
        my_ms = 1.0 + rank
        job_ms = bench.reduce_max(my_ms, world, torch.device("cpu"))
        units = bench.reduce_sum(float(w.kv_tokens()), world, torch.device("cpu"))
        results[rank] = (job_ms, units, w.query.sum().item(), w.kv_tokens())
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_time_max_and_sum_units():
    world, port = 2, _free_port()
    manager = mp.Manager()
    results = manager.dict()
    mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
    r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == 2.0                      # max over ranks
    assert r0[1] == r1[1] == r0[3] + r1[3]            # units summed over ranks
    assert r0[2] != r1[2]                             # independent batches (different seeds)
    assert r0[3] == r1[3]                             # same workload shape (fixed context lengths)
