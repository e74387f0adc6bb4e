"""The multi-rank host logic of bench.py under torch.distributed with the gloo
backend, world size 2, on CPU: the step time is the slowest rank's, the value
aggregates all ranks' work, and every rank draws its own units."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        seconds = [1.5, 2.5][rank]                     # rank 1 is the slowest
        value, slowest = bench.whole_job_tflops(1e12, 10, seconds, world)
        bench.barrier(world)
        # weak scaling: each rank's inputs come from its own seed
        w = workloads.get("tiny")
        w_rank = workloads.get("tiny", seed=w.seed + 7919 * rank)
        q = workloads.make_fwd_inputs(w_rank)["q"]
        checksum = torch.tensor([float(q.float().sum())])
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, checksum)
        out[rank] = (value, slowest, [float(g) for g in gathered])
    finally:
        dist.destroy_process_group()


def test_weak_scaling_aggregation_two_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    v0, s0, g0 = out[0]
    v1, s1, g1 = out[1]
    assert s0 == s1 == 2.5                          # max over ranks
    assert v0 == v1 == pytest.approx(2 * 1e12 * 10 / 2.5 / 1e12)
    assert g0 == g1 and g0[0] != g0[1]              # distinct units per rank
