"""Device-side failure detection, exercised without faulting, trapping or hanging a GPU.

Every wait in the library's kernels is bounded by %globaltimer; on expiry the kernel
records an error code in a device word, drains what it has in flight and returns,
and attn_get_device_status() reports ATTN_ERR_DEVICE_TIMEOUT and clears the word.
attn_selftest_timeout runs that same bounded wait on an mbarrier nothing arrives on,
with a 20 ms limit, so the timeout path runs for real.

The persistent kernels (forward, window, FP8 and decode) claim work units from one of
128 rotating counters, each tagged with its launch's generation; a launch that finds
its counter taken over by a later one stops claiming and ATTN_ERR_SCHED_CONFLICT is
reported (both launches' outputs then count as incomplete).  attn_selftest_sched drives that check on a reserved
counter; the concurrency test keeps many launches in flight on several streams and
checks that each matches a lone launch of the same call.
"""
import numpy as np
import pytest
import torch

from oracle import reference as ref
from tests.parity import check_lse, check_o, f64

pytestmark = pytest.mark.gpu

ATTN_ERR_DEVICE_TIMEOUT = -5
ATTN_ERR_SCHED_CONFLICT = -9


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


def test_expired_wait_is_reported_then_cleared(attn):
    assert attn.attn_get_device_status() == 0
    attn.attn_selftest_timeout(20_000_000)
    assert attn.attn_get_device_status() == ATTN_ERR_DEVICE_TIMEOUT
    assert attn.attn_get_device_status() == 0


def test_context_is_usable_after_a_timeout(attn):
    attn.attn_selftest_timeout(5_000_000)
    assert attn.attn_get_device_status() == ATTN_ERR_DEVICE_TIMEOUT
    g = torch.Generator().manual_seed(11)
    q, k, v = (torch.randn(1, 2, 200, 64, generator=g).to(torch.bfloat16) for _ in range(3))
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    for h in range(2):
        o_ref, lse_ref = ref.attend_head(f64(q[0, h]), f64(k[0, h]), f64(v[0, h]), 64 ** -0.5, True)
        check_o(f64(o[0, h]), o_ref, what=f"O after a timeout, head {h}")
        check_lse(f64(lse[0, h]), lse_ref)
        assert np.isfinite(f64(lse[0, h])).all()


def test_taken_over_counter_stops_the_older_launch_and_is_reported(attn):
    assert attn.attn_get_device_status() == 0
    claims = attn.attn_selftest_sched()
    assert claims == [0, 1, 2, -1, -1, 1]      # the stale claim used up generation 8's unit 0
    assert attn.attn_get_device_status() == ATTN_ERR_SCHED_CONFLICT
    assert attn.attn_get_device_status() == 0


def test_many_launches_in_flight_on_several_streams_match_lone_launches(attn):
    """96 forward/decode launches queued on 8 streams at once (under the 128 counters):
    each must equal, bit for bit, the same call run alone."""
    g = torch.Generator().manual_seed(5)
    shapes = [(1, 4, 2, 700, 128, True), (2, 2, 2, 300, 64, False), (1, 8, 8, 1500, 128, True)]
    inputs = []
    for B, Hq, Hkv, N, d, causal in shapes:
        q = torch.randn(B, Hq, N, d, generator=g).to(torch.bfloat16).cuda()
        k = torch.randn(B, Hkv, N, d, generator=g).to(torch.bfloat16).cuda()
        v = torch.randn(B, Hkv, N, d, generator=g).to(torch.bfloat16).cuda()
        inputs.append((q, k, v, causal, q[:, :, -3:].contiguous()))

    def call(i, stream=None):
        q, k, v, causal, q_last = inputs[i % len(inputs)]
        if i % 4 == 3:
            return attn.attn_decode(q_last, k, v, causal=causal, stream=stream)
        if i % 4 == 2:
            return attn.attn_fwd_window(q, k, v, window=(200, 0), stream=stream)
        return attn.attn_fwd(q, k, v, causal=causal, stream=stream)

    n = 96
    lone = []
    for i in range(n):
        lone.append(call(i))
        torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(8)]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    got = [None] * n
    for i in range(n):
        with torch.cuda.stream(streams[i % len(streams)]):
            got[i] = call(i, stream=streams[i % len(streams)])
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    for i in range(n):
        assert torch.equal(got[i][0], lone[i][0]) and torch.equal(got[i][1], lone[i][1]), i
