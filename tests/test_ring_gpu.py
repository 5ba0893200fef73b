"""Sequence-parallel ring attention: the CUDA arithmetic of the decomposition on one GPU.

Only one GPU is available to the tests, so the W ranks of the ring are emulated one
after another in one process (no kernel waits on another): for every rank, the
partials its queries compute against each K/V shard in ring order (attn_fwd, causal
on its own shard, full on earlier shards, skipped on later ones) are merged with
attn_merge, exactly as ``ring_attention_fwd`` does between its exchanges.  The
merged result of every rank must match the fp64 oracle over the whole sequence.
The backward is emulated the same way: every rank's query shard runs attn_bwd against
each K/V shard in ring order with its rows' global O and LSE, its dQ and the shards'
dK, dV summed in fp32 as ``ring_attention_bwd`` does, and all must match the oracle's
gradients over the whole sequence.  The exchange itself is tested on CPU ranks
(tests/test_ring.py).
"""
import numpy as np
import pytest
import torch

from attn_inputs import make_inputs, to_f64
from io_aware_exact_26_b200 import ring
from oracle import reference as ref
from tests.parity import check_grad, check_lse, check_o, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


@pytest.mark.parametrize("world,causal,d", [(2, True, 128), (4, True, 128), (4, False, 64), (3, True, 64)])
def test_ring_decomposition_matches_oracle(attn, world, causal, d):
    B, Hq, Hkv, n = 1, 4, 2, 384
    N = n * world
    x = make_inputs(B, Hq, Hkv, N, d, seed=100 + world + d, with_grad=False)
    q, k, v = (x[t].cuda() for t in ("q", "k", "v"))
    o_ref, lse_ref = ref.ref_fwd(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), d ** -0.5, causal)
    for r in range(world):
        sl = lambda t, s: t[:, :, s * n:(s + 1) * n].contiguous()
        qr = sl(q, r)
        o_acc = torch.zeros((B, Hq, n, d), dtype=torch.float32, device="cuda")
        lse_acc = torch.full((B, Hq, n), float("-inf"), dtype=torch.float32, device="cuda")
        out = torch.empty((B, Hq, n, d), dtype=torch.bfloat16, device="cuda")
        for step, src, kind in ring.ring_schedule(r, world, causal):
            if kind == ring.SKIP:
                continue
            o_p, lse_p = attn.attn_fwd(qr, sl(k, src), sl(v, src), causal=(kind == ring.CAUSAL))
            attn.attn_merge(o_acc, lse_acc, o_p, lse_p, out)
        torch.cuda.synchronize()
        assert attn.attn_get_device_status() == 0
        check_o(f64(out), o_ref[:, :, r * n:(r + 1) * n], f"ring W={world} rank {r} O")
        check_lse(f64(lse_acc), lse_ref[:, :, r * n:(r + 1) * n], f"ring W={world} rank {r} LSE")
        assert np.abs(f64(o_acc) - o_ref[:, :, r * n:(r + 1) * n]).max() < 1e-2


def test_merge_into_an_empty_accumulator_copies_the_partial(attn):
    rows, d = 1000, 128
    g = torch.Generator().manual_seed(3)
    o_p = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    lse_p = torch.randn(rows, generator=g).cuda()
    o_acc = torch.full((rows, d), float("nan"), device="cuda")            # ignored where lse_acc = -inf
    lse_acc = torch.full((rows,), float("-inf"), device="cuda")
    out = torch.empty((rows, d), dtype=torch.bfloat16, device="cuda")
    attn.attn_merge(o_acc, lse_acc, o_p, lse_p, out)
    torch.cuda.synchronize()
    assert torch.equal(out, o_p)
    assert torch.allclose(lse_acc, lse_p, rtol=0, atol=1e-6)


@pytest.mark.parametrize("world,causal,d", [(2, True, 128), (4, True, 128), (3, False, 64)])
def test_ring_backward_decomposition_matches_oracle(attn, world, causal, d):
    B, Hq, Hkv, n = 1, 4, 2, 320
    N = n * world
    x = make_inputs(B, Hq, Hkv, N, d, seed=200 + world + d, with_grad=True)
    q, k, v, do = (x[t].cuda() for t in ("q", "k", "v", "do"))
    sl = lambda t, s: t[:, :, s * n:(s + 1) * n].contiguous()
    dq_ref, dk_ref, dv_ref = ref.ref_bwd(*(to_f64(x[t]) for t in ("q", "k", "v", "do")), d ** -0.5, causal)
    # the forward over the ring, rank by rank: each rank's rows of O (bf16) and LSE
    o_rows, lse_rows = [], []
    for r in range(world):
        o_acc = torch.zeros((B, Hq, n, d), dtype=torch.float32, device="cuda")
        lse_acc = torch.full((B, Hq, n), float("-inf"), dtype=torch.float32, device="cuda")
        out = torch.empty((B, Hq, n, d), dtype=torch.bfloat16, device="cuda")
        for step, src, kind in ring.ring_schedule(r, world, causal):
            if kind != ring.SKIP:
                o_p, lse_p = attn.attn_fwd(sl(q, r), sl(k, src), sl(v, src), causal=(kind == ring.CAUSAL))
                attn.attn_merge(o_acc, lse_acc, o_p, lse_p, out)
        o_rows.append(out)
        lse_rows.append(lse_acc)
    # the backward over the ring: dQ per rank, dK and dV per shard, fp32 sums
    dq = [torch.zeros((B, Hq, n, d), device="cuda") for _ in range(world)]
    dkv = [torch.zeros((2, B, Hkv, n, d), device="cuda") for _ in range(world)]
    for r in range(world):
        for step, src, kind in ring.ring_schedule(r, world, causal):
            if kind == ring.SKIP:
                continue
            g = attn.attn_bwd(sl(q, r), sl(k, src), sl(v, src), o_rows[r], lse_rows[r], sl(do, r),
                              causal=(kind == ring.CAUSAL))
            dq[r] += g[0].float()
            dkv[src][0] += g[1].float()
            dkv[src][1] += g[2].float()
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    for r in range(world):
        rows = slice(r * n, (r + 1) * n)
        check_grad(f64(dq[r]), dq_ref[:, :, rows], f"ring bwd W={world} rank {r} dQ")
        check_grad(f64(dkv[r][0]), dk_ref[:, :, rows], f"ring bwd W={world} shard {r} dK")
        check_grad(f64(dkv[r][1]), dv_ref[:, :, rows], f"ring bwd W={world} shard {r} dV")
