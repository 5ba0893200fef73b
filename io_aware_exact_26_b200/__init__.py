"""Exact IO-aware attention for NVIDIA B200 (sm_100a).

The compute lives in ``libattn_b200.so`` (hand-written CUDA behind a C ABI, see
``include/attn.h``); ``binding`` marshals torch tensors into that ABI.  The
library is loaded lazily on first use, so host-side helpers such as
``accounting`` import without a GPU.
"""
from .binding import (  # noqa: F401
    AttnError,
    attn_bwd,
    attn_bwd_noalloc,
    attn_bwd_window,
    attn_decode,
    attn_decode_splits,
    attn_decode_workspace_size,
    attn_merge,
    attn_accumulate,
    NOALLOC_SCRATCH_BYTES,
    attn_bwd_workspace_size,
    attn_fwd,
    attn_fwd_fp8,
    attn_fwd_window,
    attn_get_device_status,
    attn_checks_enabled,
    attn_selftest_bounds,
    attn_selftest_sched,
    attn_selftest_timeout,
    checks_library_path,
    use_library,
    attn_status_string,
    lib,
    library_path,
)
