"""Sequence-parallel ring attention: the CUDA arithmetic of the decomposition on one GPU.

Only one GPU is available to the tests, so the W ranks of the ring are emulated one
after another in one process (no kernel waits on another): for every rank, the
partials its queries compute against each K/V shard in ring order (attn_fwd, causal
on its own shard, full on earlier shards, skipped on later ones) are merged with
attn_merge, exactly as ``ring_attention_fwd`` does between its exchanges.  The
merged result of every rank must match the fp64 oracle over the whole sequence.
The exchange itself is tested on CPU ranks (tests/test_ring.py).
"""
import numpy as np
import pytest
import torch

from attn_inputs import make_inputs, to_f64
from io_aware_exact_26_b200 import ring
from oracle import reference as ref
from tests.parity import check_lse, check_o, f64

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
