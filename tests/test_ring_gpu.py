"""Sequence-parallel ring attention: the CUDA arithmetic of the decomposition on one GPU.

Only one GPU is available to the tests, so the W ranks of the ring are emulated one
after another in one process (no kernel waits on another): for every rank, the
partials its queries compute against each K/V shard in ring order (attn_fwd, causal
on its own shard, full on earlier shards, skipped on later ones) are merged with
attn_merge, exactly as ``ring_attention_fwd`` does between its exchanges.  The
merged result of every rank must match the fp64 oracle over the whole sequence.
The backward is emulated the same way: every rank's query shard runs attn_bwd against
each K/V shard in ring order with its rows' global O and LSE, its dQ and the shards'
dK, dV summed in fp32 by attn_accumulate as ``ring_attention_bwd`` does, and all must match the oracle's
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


@pytest.mark.parametrize("n", [8, 1000, 131072 + 24])
def test_accumulate_adds_bf16_into_fp32_exactly(attn, n):
    """acc += part: bf16 to fp32 is exact, so the kernel's sum equals torch's fp32 add
    bit for bit, and a run of calls equals the same run of torch adds."""
    g = torch.Generator().manual_seed(n)
    acc = torch.randn(n, generator=g).cuda()
    parts = [torch.randn(n, generator=g).mul(10 ** k).to(torch.bfloat16).cuda() for k in range(-2, 3)]
    want = acc.clone()
    for part in parts:
        attn.attn_accumulate(acc, part)
        want += part.float()
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    assert torch.equal(acc, want)


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


@pytest.mark.parametrize("world,causal,d,layout", [(2, True, 128, "contiguous"), (4, True, 128, "contiguous"),
                                                   (3, False, 64, "contiguous"), (2, True, 128, "zigzag"),
                                                   (3, True, 64, "zigzag")])
def test_ring_backward_decomposition_matches_oracle(attn, world, causal, d, layout):
    """Forward and backward over the ring, chunk pair by chunk pair as ``ring.py`` takes
    them (both layouts), against the oracle over the whole sequence."""
    B, Hq, Hkv, c = 1, 4, 2, 192                          # c: rows per chunk
    m = len(ring.shard_chunks(0, world, layout))
    N = c * m * world
    x = make_inputs(B, Hq, Hkv, N, d, seed=200 + world + d, with_grad=True)
    q, k, v, do = (x[t].cuda() for t in ("q", "k", "v", "do"))
    ch = lambda t, a: t[:, :, a * c:(a + 1) * c].contiguous()      # global chunk a
    dq_ref, dk_ref, dv_ref = ref.ref_bwd(*(to_f64(x[t]) for t in ("q", "k", "v", "do")), d ** -0.5, causal)
    nchunks = m * world
    # forward: every query chunk's O (bf16) and LSE, merged over the key chunks
    o_ch, lse_ch = {}, {}
    for a in range(nchunks):
        o_acc = torch.zeros((B, Hq, c, d), dtype=torch.float32, device="cuda")
        lse_acc = torch.full((B, Hq, c), float("-inf"), dtype=torch.float32, device="cuda")
        out = torch.empty((B, Hq, c, d), dtype=torch.bfloat16, device="cuda")
        for b in range(nchunks):
            kind = ring.chunk_kind(a, b, causal)
            if kind != ring.SKIP:
                o_p, lse_p = attn.attn_fwd(ch(q, a), ch(k, b), ch(v, b), causal=(kind == ring.CAUSAL))
                attn.attn_merge(o_acc, lse_acc, o_p, lse_p, out)
        o_ch[a], lse_ch[a] = out, lse_acc
    # backward in ring order: rank r's chunks against the shard held at each step
    dq = {a: torch.zeros((B, Hq, c, d), device="cuda") for a in range(nchunks)}
    dkv = {a: torch.zeros((2, B, Hkv, c, d), device="cuda") for a in range(nchunks)}
    for r in range(world):
        for step in range(world):
            src = (r - step) % world
            for a in ring.shard_chunks(r, world, layout):
                for b in ring.shard_chunks(src, world, layout):
                    kind = ring.chunk_kind(a, b, causal)
                    if kind == ring.SKIP:
                        continue
                    g = attn.attn_bwd(ch(q, a), ch(k, b), ch(v, b), o_ch[a], lse_ch[a], ch(do, a),
                                      causal=(kind == ring.CAUSAL))
                    attn.attn_accumulate(dq[a], g[0])
                    attn.attn_accumulate(dkv[b][0], g[1])
                    attn.attn_accumulate(dkv[b][1], g[2])
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    for a in range(nchunks):
        rows = slice(a * c, (a + 1) * c)
        check_grad(f64(dq[a]), dq_ref[:, :, rows], f"ring bwd {layout} W={world} chunk {a} dQ")
        check_grad(f64(dkv[a][0]), dk_ref[:, :, rows], f"ring bwd {layout} W={world} chunk {a} dK")
        check_grad(f64(dkv[a][1]), dv_ref[:, :, rows], f"ring bwd {layout} W={world} chunk {a} dV")
