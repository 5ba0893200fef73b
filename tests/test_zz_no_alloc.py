"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc -- code embedded in a host framework whose pool
owns all device memory, or a loop that must not allocate once it runs -- so the
library offers a backward whose scratch is its own fixed device array.  This file
is collected last on purpose: it checks, through the C ABI, that two calls in a
row give bit-for-bit the gradients of attn_bwd with a caller-allocated workspace
(the backward's reduction order is fixed, so the bits must agree), that the second
call leaves the device's free memory and torch's allocated bytes unchanged, and
that shapes too large for the fixed array are refused before anything is launched.
"""
import pytest
import torch

from attn_inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [(1, 4, 2, 1000, 128, True), (2, 2, 2, 384, 64, False)])
def test_noalloc_matches_workspace_backward_twice(attn, B, Hq, Hkv, N, d, causal):
    assert attn.attn_bwd_workspace_size(B, Hq, Hkv, N, d, causal) <= attn.NOALLOC_SCRATCH_BYTES
    x = make_inputs(B, Hq, Hkv, N, d, seed=4242 + N)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.attn_fwd(q, k, v, causal=causal)
    ws = torch.empty(attn.attn_bwd_workspace_size(B, Hq, Hkv, N, d, causal), dtype=torch.uint8, device="cuda")
    ref = attn.attn_bwd(q, k, v, o, lse, do, causal=causal, workspace=ws)
    torch.cuda.synchronize()
    for call in range(2):
        outs = (torch.full_like(q, float("nan")), torch.full_like(k, float("nan")), torch.full_like(v, float("nan")))
        torch.cuda.synchronize()
        free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        attn.attn_bwd_noalloc(q, k, v, o, lse, do, *outs, causal=causal)
        torch.cuda.synchronize()
        free1, alloc1 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        assert attn.attn_get_device_status() == 0
        if call == 1:   # the first call may still load the module / look up the array
            assert free1 == free0 and alloc1 == alloc0
        for got, want, name in zip(outs, ref, ("dQ", "dK", "dV")):
            assert torch.equal(got, want), name


def test_noalloc_rejects_shapes_beyond_its_scratch(attn):
    B, Hq, Hkv, N, d = 64, 32, 8, 8192, 128
    assert attn.attn_bwd_workspace_size(B, Hq, Hkv, N, d, True) > attn.NOALLOC_SCRATCH_BYTES
    q = torch.empty((1,), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1,), dtype=torch.float32, device="cuda")
    p = q.data_ptr()
    st = attn.lib().attn_bwd_noalloc(p, p, p, p, lse.data_ptr(), p, p, p, p, B, Hq, Hkv, N, d, 0.088, 1,
                                     torch.cuda.current_stream().cuda_stream)
    assert st == -6   # ATTN_ERR_WORKSPACE, nothing launched
