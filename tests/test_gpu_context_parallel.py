"""Context-parallel forward on one GPU.

A one-rank NCCL group runs the whole product path (the all-gather, then the
rank-order fold) against the oracle.  With more ranks every rank computes the
fold of the gathered shards in rank order; that fold, with the shards
gathered by stacking, is checked against the oracle on the concatenated K/V
and for bitwise repeatability.  (Runs with several GPUs exchanging shards are
not possible on a one-GPU machine; the gather's ordering is covered by the
two-rank gloo test in test_multiproc.py.)

Bars as for the bf16 forward: max |dO| <= 2e-2, max |dLSE| <= 1e-3.
"""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from parity import LSE_MAX_ABS, O_MAX_ABS, O_NRMS, fwd_errors, oracle_fwd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import head_attention_qk_b200 as pkg

    return pkg


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(seed, B, Hq, Hkv, Sq, shard_len, world):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, Sq, 128, generator=g).to(torch.bfloat16)
    ks = [torch.randn(B, Hkv, shard_len, 128, generator=g).to(torch.bfloat16) for _ in range(world)]
    vs = [torch.randn(B, Hkv, shard_len, 128, generator=g).to(torch.bfloat16) for _ in range(world)]
    return q, ks, vs


def test_context_parallel_one_rank_nccl(h):
    q, ks, vs = _inputs(41, 1, 4, 2, 300, 700, 1)
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % _port(), rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        out, lse = h.attn_fwd_context_parallel(q.cuda(), ks[0].cuda(), vs[0].cuda())
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert h.get_device_error() == 0
    o_ref, lse_ref = oracle_fwd(q, ks[0], vs[0], 1.0 / np.sqrt(128))
    e = fwd_errors(out, lse, o_ref, lse_ref)
    assert e["o_max_abs"] <= O_MAX_ABS and e["lse_max_abs"] <= LSE_MAX_ABS and e["o_nrms"] <= O_NRMS, e


@pytest.mark.parametrize("world,shard_len", [(2, 640), (4, 333), (8, 129)])
def test_rank_order_fold_of_gathered_shards(h, world, shard_len):
    q, ks, vs = _inputs(50 + world, 2, 8, 2, 257, shard_len, world)
    kg = torch.stack(ks).cuda()                      # what the all-gather leaves on every rank
    vg = torch.stack(vs).cuda()
    runs = [h.attn_fwd_kvblocks(q.cuda(), [kg[r] for r in range(world)], [vg[r] for r in range(world)])
            for _ in range(2)]
    assert h.get_device_error() == 0
    assert torch.equal(runs[0][0].view(torch.int16), runs[1][0].view(torch.int16))
    assert torch.equal(runs[0][1].view(torch.int32), runs[1][1].view(torch.int32))
    o_ref, lse_ref = oracle_fwd(q, torch.cat(ks, dim=2), torch.cat(vs, dim=2), 1.0 / np.sqrt(128))
    e = fwd_errors(runs[0][0], runs[0][1], o_ref, lse_ref)
    assert e["o_max_abs"] <= O_MAX_ABS and e["lse_max_abs"] <= LSE_MAX_ABS and e["o_nrms"] <= O_NRMS, e
