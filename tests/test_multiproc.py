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


def _cp_worker(rank, world, port, out):
    import datetime
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from head_attention_qk_b200.context_parallel import attn_fwd_context_parallel, gather_kv_shards

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r's shard holds the value 100 r + position, so the gathered order is visible
        k = (torch.arange(2 * 3 * 5 * 4, dtype=torch.float32).view(2, 3, 5, 4) + 100 * rank)
        v = -k
        kg, vg = gather_kv_shards(k, v)
        ok = kg.shape == (world, 2, 3, 5, 4) and all(
            torch.equal(kg[r], k - 100 * rank + 100 * r) and torch.equal(vg[r], -kg[r]) for r in range(world))
        # shards of different lengths are refused on every rank (no rank is left waiting)
        k2 = torch.zeros(1, 1, 3 + rank, 4)
        try:
            gather_kv_shards(k2, k2)
            refused = False
        except ValueError:
            refused = True
        # the attention itself runs only in the CUDA library: CPU tensors are
        # refused after the exchange (the same steps on every rank), never computed
        q = torch.zeros(1, 2, 8, 128, dtype=torch.bfloat16)
        kv = torch.zeros(1, 2, 6, 128, dtype=torch.bfloat16)
        try:
            attn_fwd_context_parallel(q, kv, kv)
            no_fallback = False
        except ValueError as e:
            no_fallback = "CUDA" in str(e)
        out[rank] = (ok, refused, no_fallback)
    finally:
        dist.destroy_process_group()


def test_context_parallel_gather_order_two_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    mp.start_processes(_cp_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == (True, True, True) and out[1] == (True, True, True)
