"""Sequence-parallel ring attention: the host logic on CPU ranks (gloo), no GPU.

Each rank holds one contiguous shard of Q, K, V; the K/V shards travel around the
ring and every partial is merged by its log-sum-exp.  Here the partial attention is
the fp64 oracle and the merge a plain fp64 restatement of the LSE rescale, so the
test checks the ring's schedule, its point-to-point exchange and the merge order:
the result on every rank must equal the oracle's attention over the whole sequence.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from io_aware_exact_26_b200 import ring
from oracle import reference as ref


def test_schedule_covers_every_shard_once_and_masks_causally():
    for world in (1, 2, 3, 5):
        for rank in range(world):
            sch = ring.ring_schedule(rank, world, causal=True)
            assert sorted(src for _, src, _ in sch) == list(range(world))
            for _, src, kind in sch:
                assert kind == (ring.CAUSAL if src == rank else ring.FULL if src < rank else ring.SKIP)
            assert all(kind == ring.FULL for _, _, kind in ring.ring_schedule(rank, world, causal=False))


def _partial(q, k, v, causal, scale):
    o, lse = ref.ref_fwd(q.numpy(), k.numpy(), v.numpy(), scale, causal)
    return torch.from_numpy(o), torch.from_numpy(lse)


def _merge(o_acc, lse_acc, o_p, lse_p):
    m = torch.maximum(lse_acc, lse_p)
    a = torch.where(torch.isinf(lse_acc), torch.zeros_like(m), torch.exp(lse_acc - m))
    b = torch.where(torch.isinf(lse_p), torch.zeros_like(m), torch.exp(lse_p - m))
    o_acc.copy_((a[..., None] * o_acc + b[..., None] * o_p) / (a + b)[..., None])
    lse_acc.copy_(m + torch.log(a + b))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, causal, shape, out_dir, layout="contiguous"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hkv, N, d = shape
        g = torch.Generator().manual_seed(1234)            # the same full problem on every rank
        q, k, v = (torch.randn(B, h, N, d, generator=g, dtype=torch.float64) for h in (Hq, Hkv, Hkv))
        shard = lambda t: ring.shard_sequence(t, rank, world, layout)
        o, lse = ring.ring_attention_fwd(shard(q), shard(k), shard(v), causal=causal, scale=0.4,
                                         partial=_partial, merge=_merge, acc_dtype=torch.float64, layout=layout)
        np.save(os.path.join(out_dir, f"o{rank}.npy"), o.numpy())
        np.save(os.path.join(out_dir, f"lse{rank}.npy"), lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout", [(2, "contiguous"), (3, "contiguous"), (2, "zigzag"), (3, "zigzag")])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_equals_attention_over_the_whole_sequence(tmp_path, world, layout, causal):
    shape = (2, 4, 2, 12 * world, 5)
    mp.start_processes(_rank_main, args=(world, _free_port(), causal, shape, str(tmp_path), layout), nprocs=world,
                       join=True, start_method="spawn")
    B, Hq, Hkv, N, d = shape
    g = torch.Generator().manual_seed(1234)
    q, k, v = (torch.randn(B, h, N, d, generator=g, dtype=torch.float64).numpy() for h in (Hq, Hkv, Hkv))
    o_ref, lse_ref = ref.ref_fwd(q, k, v, 0.4, causal)
    for r in range(world):
        mine = lambda a, dim: ring.shard_sequence(torch.from_numpy(a), r, world, layout, dim).numpy()
        np.testing.assert_allclose(np.load(tmp_path / f"o{r}.npy"), mine(o_ref, 2), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(np.load(tmp_path / f"lse{r}.npy"), mine(lse_ref, 2), rtol=1e-12, atol=1e-13)


def test_shards_partition_the_sequence_and_zigzag_balances_causal_work():
    for world in (1, 2, 3, 4, 8):
        for layout in ring.LAYOUTS:
            held = sorted(a for r in range(world) for a in ring.shard_chunks(r, world, layout))
            assert held == list(range(world * len(ring.shard_chunks(0, world, layout))))
            x = torch.arange(2 * world * 3).reshape(1, 1, -1, 1)
            got = torch.cat([ring.shard_sequence(x, r, world, layout) for r in range(world)], dim=2)
            assert sorted(got.flatten().tolist()) == x.flatten().tolist()
        # causal work per rank, counting a diagonal chunk pair as half a full one
        work = lambda r, layout: sum(
            {ring.FULL: 1.0, ring.CAUSAL: 0.5, ring.SKIP: 0.0}[ring.chunk_kind(a, b, True)]
            for a in ring.shard_chunks(r, world, layout)
            for s in range(world) for b in ring.shard_chunks(s, world, layout))
        assert len({work(r, "zigzag") for r in range(world)}) == 1
        if world > 1:
            assert work(world - 1, "contiguous") > work(0, "contiguous")


def _partial_bwd(q, k, v, o, lse, do, causal, scale):
    """One shard pair's gradient contribution in fp64, with the rows' global O and LSE:
    P = exp(scale q k^T - lse), D = rowsum(dO * O), dS = P (dO v^T - D)."""
    G = q.shape[1] // k.shape[1]
    kk, vv = k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1)
    s = scale * q @ kk.transpose(-1, -2)
    if causal:
        n = q.shape[2]
        s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    p = torch.exp(s - lse[..., None])
    ds = p * (do @ vv.transpose(-1, -2) - (do * o).sum(-1, keepdim=True))
    dq = scale * ds @ kk
    B, Hkv, n, d = k.shape
    dk = (scale * ds.transpose(-1, -2) @ q).reshape(B, Hkv, G, n, d).sum(2)
    dv = (p.transpose(-1, -2) @ do).reshape(B, Hkv, G, n, d).sum(2)
    return dq, dk, dv


def _accumulate(acc, part):
    acc += part.to(acc.dtype)


def _rank_bwd(rank, world, port, causal, shape, out_dir, layout="contiguous"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hkv, N, d = shape
        g = torch.Generator().manual_seed(4321)            # the same full problem on every rank
        q, k, v = (torch.randn(B, h, N, d, generator=g, dtype=torch.float64) for h in (Hq, Hkv, Hkv))
        do = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64)
        shard = lambda t: ring.shard_sequence(t, rank, world, layout)
        o, lse = ring.ring_attention_fwd(shard(q), shard(k), shard(v), causal=causal, scale=0.4,
                                         partial=_partial, merge=_merge, acc_dtype=torch.float64, layout=layout)
        dq, dk, dv = ring.ring_attention_bwd(shard(q), shard(k), shard(v), o, lse, shard(do), causal=causal,
                                             scale=0.4, partial=_partial_bwd, accumulate=_accumulate,
                                             acc_dtype=torch.float64, layout=layout)
        for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            np.save(os.path.join(out_dir, f"{name}{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout", [(2, "contiguous"), (3, "contiguous"), (4, "contiguous"),
                                          (2, "zigzag"), (3, "zigzag")])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_backward_equals_gradients_over_the_whole_sequence(tmp_path, world, layout, causal):
    """Every rank's dQ and the dK, dV its shards collect on their way round the ring
    equal the oracle's gradients over the whole sequence (GQA, group of 2)."""
    shape = (2, 4, 2, 8 * world, 5)
    mp.start_processes(_rank_bwd, args=(world, _free_port(), causal, shape, str(tmp_path), layout), nprocs=world,
                       join=True, start_method="spawn")
    B, Hq, Hkv, N, d = shape
    g = torch.Generator().manual_seed(4321)
    q, k, v = (torch.randn(B, h, N, d, generator=g, dtype=torch.float64).numpy() for h in (Hq, Hkv, Hkv))
    do = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64).numpy()
    grads = dict(zip(("dq", "dk", "dv"), ref.ref_bwd(q, k, v, do, 0.4, causal)))
    for r in range(world):
        for name, full in grads.items():
            mine = ring.shard_sequence(torch.from_numpy(full), r, world, layout).numpy()
            np.testing.assert_allclose(np.load(tmp_path / f"{name}{r}.npy"), mine,
                                       rtol=1e-10, atol=1e-11, err_msg=f"{name} rank {r}")


@pytest.mark.parametrize("world,causal,layout", [(2, True, "zigzag"), (4, True, "zigzag"), (8, True, "zigzag"),
                                                 (3, True, "contiguous"), (4, False, "contiguous")])
def test_rank_chunk_pairs_cover_every_visible_pair_once(world, causal, layout):
    """Over all ranks the ring computes every (query chunk, key chunk) pair the mask leaves
    visible exactly once, each at the step its key chunk is held, with the right kind."""
    nch = world * len(ring.shard_chunks(0, world, layout))
    seen = []
    for r in range(world):
        for step, i, a, j, b, kind in ring.rank_chunk_pairs(r, world, causal, layout):
            assert ring.shard_chunks(r, world, layout)[i] == a
            assert ring.shard_chunks((r - step) % world, world, layout)[j] == b
            assert kind == (ring.CAUSAL if causal and a == b else ring.FULL)
            seen.append((a, b))
    want = [(a, b) for a in range(nch) for b in range(nch) if not causal or b <= a]
    assert sorted(seen) == sorted(want)


def test_ring_step_bytes_of_the_long_causal_workload():
    import bench
    w = bench.WORKLOADS["long_causal_b1_h32_n32768_d128"]
    sb = bench.ring_step_bytes(w, 4, "zigzag")
    rows = 32768 // 4
    assert sb["chunks_per_shard"] == 2
    assert sb["fwd"] == 2 * 32 * rows * 128 * 2                 # K and V of the shard, bf16
    assert sb["bwd"] == sb["fwd"] + 2 * 32 * rows * 128 * 4     # plus its fp32 dK, dV accumulators
