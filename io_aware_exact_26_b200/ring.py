"""Sequence-parallel (context-parallel) attention forward over a ring of ranks.

Page "attention 的显存线性化" §五 names sequence parallelism among the later
FlashAttention versions' features; the pages give no algorithm for it, so this
follows the plainest reading that the rest of the pages support: a sequence too
long for one GPU is cut into W contiguous shards, one per rank, and the online
softmax (page "attn-efficient", online-softmax section) is applied to whole K/V
shards instead of tiles.

Rank r holds positions [r*n, (r+1)*n) of Q, K and V (n = N / W).  In W steps the
K/V shards travel around the ring: at step s rank r holds the shard that started on
rank (r - s) mod W, computes the attention of its own queries against it -- a
partial (O_s, LSE_s) -- and merges that into a running (O, LSE) with the LSE
rescale.  Meanwhile the shard for step s+1 is already in flight: each rank sends
its current shard to rank r+1 and receives the next from rank r-1.  Under causal
masking, shards from later positions are skipped, the rank's own shard is causal
and earlier shards are seen in full.

B200 notes.  Remote K/V always land in a local buffer first (point-to-point sends
of the communication backend, NCCL over NVLink on GPUs), so no kernel reads another
GPU's memory; the transfer of the next shard overlaps the compute of the current
one.  Every rank takes the same W - 1 exchange steps in the same order, skipped
compute included.  Only the forward is provided.

The partial and merge steps are parameters: on GPUs they are ``attn_fwd`` and
``attn_merge`` of the CUDA library (the defaults); tests pass other functions to
check the ring logic on CPU ranks.
"""
from __future__ import annotations

import torch

FULL, CAUSAL, SKIP = "full", "causal", "skip"


def ring_schedule(rank: int, world: int, causal: bool):
    """[(step, source rank, kind)] for one rank: the shard it holds at each step and
    what it computes against it."""
    out = []
    for s in range(world):
        src = (rank - s) % world
        if not causal:
            kind = FULL
        elif src == rank:
            kind = CAUSAL
        elif src < rank:
            kind = FULL
        else:
            kind = SKIP
        out.append((s, src, kind))
    return out


def _cuda_partial(q, k, v, causal, scale):
    from . import binding
    return binding.attn_fwd(q, k, v, scale=scale, causal=causal)


def _cuda_merge(o_acc, lse_acc, o_part, lse_part):
    from . import binding
    binding.attn_merge(o_acc, lse_acc, o_part, lse_part)


def ring_attention_fwd(q, k, v, *, causal: bool, group=None, scale=None, partial=None, merge=None,
                       acc_dtype=torch.float32):
    """Attention of this rank's query shard against the whole sequence.

    q: [B, Hq, n, d]; k, v: [B, Hkv, n, d] -- this rank's shard (all ranks the same n).
    Returns (o, lse): o [B, Hq, n, d] and lse [B, Hq, n] (natural log) in ``acc_dtype``
    (fp32 by default: merged in fp32, cast as needed).
    ``partial(q, k, v, causal, scale) -> (o, lse)`` and ``merge(o_acc, lse_acc, o_part,
    lse_part)`` (in place) default to the CUDA library.
    """
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    partial = partial or _cuda_partial
    merge = merge or _cuda_merge
    if scale is None:
        scale = q.shape[-1] ** -0.5
    B, Hq, n, d = q.shape
    o_acc = torch.zeros((B, Hq, n, d), dtype=acc_dtype, device=q.device)
    lse_acc = torch.full((B, Hq, n), float("-inf"), dtype=acc_dtype, device=q.device)
    cur = torch.stack((k, v)).contiguous()          # [2, B, Hkv, n, d]: one message per step
    nxt = torch.empty_like(cur)
    nxt_rank = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv_rank = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    for step, src, kind in ring_schedule(rank, world, causal):
        reqs = []
        if step + 1 < world:                        # post the exchange for the next step first
            ops = [dist.P2POp(dist.isend, cur, nxt_rank, group), dist.P2POp(dist.irecv, nxt, prv_rank, group)]
            reqs = dist.batch_isend_irecv(ops)
        if kind != SKIP:
            o_p, lse_p = partial(q, cur[0], cur[1], kind == CAUSAL, scale)
            merge(o_acc, lse_acc, o_p, lse_p)
        for r in reqs:
            r.wait()
        if step + 1 < world:
            cur, nxt = nxt, cur
    return o_acc, lse_acc
