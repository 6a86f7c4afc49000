"""B200 (sm_100a) hashed n-gram (PLE / Engram) embedding lookup.

The C ABI is in include/ple.h; libple.so is built in-tree from csrc/ by
``_build.build()``.  This package is a thin binding over it.
"""
from .binding import (  # noqa: F401
    PLE_BF16, PLE_ERR_BAD_ROW, PLE_ERR_BAD_SEQLENS, PLE_F32, PLE_F8E4M3, PLE_OK, Plan, PleError, alloc_workspace, lib,
    ple_gather, ple_grad_scatter, ple_grad_scatter_atomic, ple_grad_scatter_noalloc, ple_hash, ple_lookup,
    ple_lookup_slice, ple_status, workspace_bytes, conv_forward, conv_backward, conv_workspace_bytes, Prefetched,
    ple_prefetch, ple_gather_cache, ple_grad_scatter_cache, ple_grad_prepare, ple_grad_apply, PLE_ERR_TIMEOUT,
    set_wait_limit_ns, default_wait_limit_ns, noalloc_scratch_bytes)
