"""Device-side failure detection, exercised without faulting, trapping or hanging a GPU.

Every wait in the library's kernels is bounded by %globaltimer; on expiry the kernel
records an error code in a device word, drains what it has in flight and returns,
and attn_get_device_status() reports ATTN_ERR_DEVICE_TIMEOUT and clears the word.
attn_selftest_timeout runs that same bounded wait on an mbarrier nothing arrives on,
with a 20 ms limit, so the timeout path runs for real.
"""
import numpy as np
import pytest
import torch

from oracle import reference as ref
from tests.parity import check_lse, check_o, f64

pytestmark = pytest.mark.gpu

ATTN_ERR_DEVICE_TIMEOUT = -5


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
