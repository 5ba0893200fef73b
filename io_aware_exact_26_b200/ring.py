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
one.  Every rank takes the same exchange steps in the same order, skipped compute
included.

Layouts.  ``contiguous``: rank r holds chunk r of W equal chunks, as above; under
causal masking rank r then does r + 1 of the W shard pairs' work.  ``zigzag``: the
sequence is cut into 2W chunks and rank r holds chunks r and 2W - 1 - r (in that
order, as one local tensor); every rank then does the same causal work, 2W - 1 full
chunk pairs and 2 diagonal ones.  Chunk pairs are computed one by one: full where
the key chunk precedes the query chunk, causal on the diagonal, skipped after it.

Backward (recompute, as on one GPU): the shards travel the same ring, each with
fp32 accumulators for its dK and dV.  At step s rank r computes the gradient
contributions of its query shard against the shard it holds -- with the global LSE
and O of its rows from the forward, the probabilities and D = rowsum(dO * O) are
those of the whole sequence -- adds dQ to its own accumulator and dK, dV to the
travelling ones, and passes them on.  After the last step one more hop brings every
shard's accumulators back to their owner.

The partial and merge steps are parameters: on GPUs they are ``attn_fwd``,
``attn_merge`` and ``attn_bwd`` of the CUDA library (the defaults); tests pass other
functions to check the ring logic on CPU ranks.
"""
from __future__ import annotations

import torch

FULL, CAUSAL, SKIP = "full", "causal", "skip"
LAYOUTS = ("contiguous", "zigzag")


def ring_schedule(rank: int, world: int, causal: bool):
    """[(step, source rank, kind)] for one rank under the contiguous layout: the shard
    it holds at each step and what it computes against it."""
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


def shard_chunks(rank: int, world: int, layout: str = "contiguous"):
    """Global chunk indices held by ``rank``, in local order (chunks of N / W positions
    for ``contiguous``, of N / (2W) for ``zigzag``)."""
    if layout == "contiguous":
        return [rank]
    if layout == "zigzag":
        return [rank, 2 * world - 1 - rank]
    raise ValueError(f"layout must be one of {LAYOUTS}")


def chunk_kind(a: int, b: int, causal: bool):
    """What query chunk a computes against key chunk b."""
    if not causal or b < a:
        return FULL
    return CAUSAL if a == b else SKIP


def rank_chunk_pairs(rank: int, world: int, causal: bool, layout: str = "contiguous"):
    """[(step, i, a, j, b, kind)]: at ring step ``step`` this rank's local chunk i (global
    chunk a) against local chunk j (global chunk b) of the shard it then holds, skipped
    pairs left out -- the pairs ``ring_attention_fwd`` and ``ring_attention_bwd`` compute,
    in their order."""
    out = []
    mine = shard_chunks(rank, world, layout)
    for step in range(world):
        src = (rank - step) % world
        for i, a in enumerate(mine):
            for j, b in enumerate(shard_chunks(src, world, layout)):
                kind = chunk_kind(a, b, causal)
                if kind != SKIP:
                    out.append((step, i, a, j, b, kind))
    return out


def shard_sequence(x, rank: int, world: int, layout: str = "contiguous", dim: int = 2):
    """This rank's local tensor of a full-sequence tensor ``x`` (sequence along ``dim``)."""
    chunks = shard_chunks(rank, world, layout)
    nchunks = world * len(chunks)
    c = x.shape[dim] // nchunks
    if c * nchunks != x.shape[dim]:
        raise ValueError(f"sequence length {x.shape[dim]} is not a multiple of {nchunks} chunks")
    return torch.cat([x.narrow(dim, a * c, c) for a in chunks], dim=dim).contiguous()


def _chunked(x, m):
    """[B, H, m*c, d] -> [m, B, H, c, d] (each chunk contiguous)."""
    B, H, n, d = x.shape
    return x.reshape(B, H, m, n // m, d).permute(2, 0, 1, 3, 4).contiguous()


def _unchunked(x):
    """[m, B, H, c, ...] -> [B, H, m*c, ...]."""
    return torch.cat(list(x.unbind(0)), dim=2)


def _cuda_partial(q, k, v, causal, scale):
    from . import binding
    return binding.attn_fwd(q, k, v, scale=scale, causal=causal)


def _cuda_merge(o_acc, lse_acc, o_part, lse_part):
    from . import binding
    binding.attn_merge(o_acc, lse_acc, o_part, lse_part)


def _ring_peers(group, rank, world):
    import torch.distributed as dist
    if group is None:
        return (rank + 1) % world, (rank - 1) % world
    return dist.get_global_rank(group, (rank + 1) % world), dist.get_global_rank(group, (rank - 1) % world)


def ring_attention_fwd(q, k, v, *, causal: bool, group=None, scale=None, partial=None, merge=None,
                       acc_dtype=torch.float32, layout: str = "contiguous"):
    """Attention of this rank's query shard against the whole sequence.

    q: [B, Hq, n, d]; k, v: [B, Hkv, n, d] -- this rank's shard (all ranks the same n;
    under ``zigzag`` the rank's two chunks, in order, see ``shard_sequence``).
    Returns (o, lse): o [B, Hq, n, d] and lse [B, Hq, n] (natural log) in ``acc_dtype``
    (fp32 by default: merged in fp32, cast as needed), rows in the shard's order.
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
    mine = shard_chunks(rank, world, layout)
    m = len(mine)
    B, Hq, n, d = q.shape
    qc = _chunked(q, m)                                       # [m, B, Hq, c, d]
    o_acc = torch.zeros((m, B, Hq, n // m, d), dtype=acc_dtype, device=q.device)
    lse_acc = torch.full((m, B, Hq, n // m), float("-inf"), dtype=acc_dtype, device=q.device)
    cur = torch.stack((_chunked(k, m), _chunked(v, m))).contiguous()   # [2, m, B, Hkv, c, d]: one message
    nxt = torch.empty_like(cur)
    nxt_rank, prv_rank = _ring_peers(group, rank, world)
    pairs = rank_chunk_pairs(rank, world, causal, layout)
    for step in range(world):
        reqs = []
        if step + 1 < world:                        # post the exchange for the next step first
            ops = [dist.P2POp(dist.isend, cur, nxt_rank, group), dist.P2POp(dist.irecv, nxt, prv_rank, group)]
            reqs = dist.batch_isend_irecv(ops)
        for _, i, _, j, _, kind in (pr for pr in pairs if pr[0] == step):
            o_p, lse_p = partial(qc[i], cur[0, j], cur[1, j], kind == CAUSAL, scale)
            merge(o_acc[i], lse_acc[i], o_p, lse_p)
        for r in reqs:
            r.wait()
        if step + 1 < world:
            cur, nxt = nxt, cur
    return _unchunked(o_acc), _unchunked(lse_acc[..., None])[..., 0]


def _cuda_partial_bwd(q, k, v, o, lse, do, causal, scale):
    from . import binding
    return binding.attn_bwd(q, k, v, o, lse, do, scale=scale, causal=causal)


def _cuda_accumulate(acc, part):
    from . import binding
    binding.attn_accumulate(acc, part)


def ring_attention_bwd(q, k, v, o, lse, do, *, causal: bool, group=None, scale=None, partial=None,
                       accumulate=None, acc_dtype=torch.float32, layout: str = "contiguous"):
    """Gradients of this rank's shards, for attention over the whole ring's sequence.

    q, o, do: [B, Hq, n, d]; k, v: [B, Hkv, n, d] -- this rank's shard; lse: [B, Hq, n]
    (natural log), o and lse being this rank's rows of the forward over the whole
    sequence (``ring_attention_fwd`` with the same layout; o in the dtype ``partial``
    takes).  Returns (dq, dk, dv) for this rank's shards in ``acc_dtype``.
    ``partial(q, k, v, o, lse, do, causal, scale) -> (dq, dk, dv)`` gives one chunk
    pair's contribution and ``accumulate(acc, part)`` adds one into an accumulator in
    place; they default to the CUDA library's ``attn_bwd`` and ``attn_accumulate``
    (fp32 accumulators, ``acc_dtype`` torch.float32).
    """
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    partial = partial or _cuda_partial_bwd
    accumulate = accumulate or _cuda_accumulate
    if scale is None:
        scale = q.shape[-1] ** -0.5
    mine = shard_chunks(rank, world, layout)
    m = len(mine)
    qc, oc, doc = _chunked(q, m), _chunked(o, m), _chunked(do, m)
    lsec = _chunked(lse[..., None], m)[..., 0]
    dq = torch.zeros(qc.shape, dtype=acc_dtype, device=q.device)
    cur = torch.stack((_chunked(k, m), _chunked(v, m))).contiguous()   # the shard held at this step
    nxt = torch.empty_like(cur)
    acc = torch.zeros(cur.shape, dtype=acc_dtype, device=q.device)      # its dK, dV so far
    acc_in = torch.empty_like(acc)
    nxt_rank, prv_rank = _ring_peers(group, rank, world)
    pairs = rank_chunk_pairs(rank, world, causal, layout)
    for step in range(world):
        reqs = []
        if step + 1 < world:                        # the next shard is in flight during the compute
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, cur, nxt_rank, group),
                                           dist.P2POp(dist.irecv, nxt, prv_rank, group)])
        for _, i, _, j, _, kind in (pr for pr in pairs if pr[0] == step):
            dq_p, dk_p, dv_p = partial(qc[i], cur[0, j], cur[1, j], oc[i], lsec[i], doc[i], kind == CAUSAL, scale)
            accumulate(dq[i], dq_p)
            accumulate(acc[0, j], dk_p)
            accumulate(acc[1, j], dv_p)
        # this shard's accumulators move on with it (the last hop brings them home)
        if world > 1:
            reqs += dist.batch_isend_irecv([dist.P2POp(dist.isend, acc, nxt_rank, group),
                                            dist.P2POp(dist.irecv, acc_in, prv_rank, group)])
        for r in reqs:
            r.wait()
        if world > 1:
            acc, acc_in = acc_in, acc
        if step + 1 < world:
            cur, nxt = nxt, cur
    return _unchunked(dq), _unchunked(acc[0]), _unchunked(acc[1])
