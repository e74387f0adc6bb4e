"""Context-parallel (sequence-parallel) forward over ranks of a torch.distributed
process group.

Each rank holds its own query rows and one shard of the keys and values; the
shards of all ranks, in rank order, form the whole K/V.  The exchange step is
an all-gather of the K/V shards into this GPU's memory (NCCL between GPUs),
after which every rank attends to the gathered blocks in rank order with
``attn_fwd_kvblocks``: one launch folds up to 32 blocks tile by tile in that
fixed order (the LSE merge rule), so a rank's output does not depend on
timing or on which rank finished first.

Pages: FlashDreams issue #739 ("[Proposal] ROCm (AMD Instinct) support for the
core attention and distributed init"), on its ContextParallelAttention path,
which combines per-shard attention through the log-sum-exp, and on Ulysses K/V
traffic; RL-Kernel PR #319 ("feat(attention): add strict bitwise ROCm path"),
table "Distributed (strict CP, RCCL AG+RS)": context parallelism by
all-gather with bitwise-stable results.

Shards must have the same length on every rank (the gathered buffer is then
one contiguous [world, B, Hkv, L, D] tensor whose slices are the blocks); a
mismatch is refused on every rank.  bf16 only, like attn_fwd_kvblocks.
"""
import torch
import torch.distributed as dist

from . import hattn


def gather_kv_shards(k, v, group=None):
    """All-gather this rank's K and V shards ([B, Hkv, L, D], the same shape on
    every rank) into two [world, B, Hkv, L, D] tensors; index r is rank r's
    shard.  Runs on torch's current stream (NCCL) or on the host (gloo)."""
    if k.shape != v.shape or k.dim() != 4:
        raise ValueError("k and v must be [B, Hkv, L, D] shards of the same shape")
    world = dist.get_world_size(group)
    shape = torch.tensor(list(k.shape), dtype=torch.int64, device=k.device)
    shapes = [torch.empty_like(shape) for _ in range(world)]
    dist.all_gather(shapes, shape, group=group)
    if any(not torch.equal(s, shape) for s in shapes):
        raise ValueError("every rank must hold K/V shards of the same shape: %s"
                         % [tuple(int(x) for x in s.tolist()) for s in shapes])
    kg = torch.empty((world,) + tuple(k.shape), dtype=k.dtype, device=k.device)
    vg = torch.empty_like(kg)
    # gathered along the first dimension: [world * B, Hkv, L, D] views of the buffers
    flat = (world * k.shape[0],) + tuple(k.shape[1:])
    dist.all_gather_into_tensor(kg.view(flat), k.contiguous(), group=group)
    dist.all_gather_into_tensor(vg.view(flat), v.contiguous(), group=group)
    return kg, vg


def attn_fwd_context_parallel(q, k, v, group=None, scale=None, out=None, lse=None, stream=None):
    """O [B, Hq, Sq, D] bf16 and LSE [B, Hq, Sq] fp32 of this rank's queries q
    against the K/V shards of all ranks of ``group`` (this rank's k, v
    [B, Hkv, L, D]), folded in rank order.  The all-gather runs on torch's
    current stream; with a ``stream`` of the caller's, the attention kernel
    waits there for the gather, and the gathered buffers stay reserved for
    that stream until its work on them is done."""
    kg, vg = gather_kv_shards(k, v, group)
    world = kg.shape[0]
    if stream is not None and kg.is_cuda:
        cur = torch.cuda.current_stream(kg.device)
        if stream != cur:
            stream.wait_stream(cur)
            kg.record_stream(stream)
            vg.record_stream(stream)
    return hattn.attn_fwd_kvblocks(q, [kg[r] for r in range(world)], [vg[r] for r in range(world)], scale=scale,
                                   out=out, lse=lse, stream=stream)
