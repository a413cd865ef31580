"""Shared-prefix attention over a flat, deduplicated packed layout, for B200.

The compute path is libpsa.so (hand-written sm_100a CUDA behind a C ABI,
declared in include/psa.h); this package is its thin ctypes binding plus the
seeded workload generators.  The library is loaded on first use and a
missing build raises -- there is no CPU fallback.
"""
from ._binding import (  # noqa: F401
    EXPORTS, LIB_PATH, DEBUG_LIB_PATH, use_library, PsaError, Rect, Segment, VerifyFeatures, KvScales, build_schedule,
    build_spec,
    lib, plan_prefill, prefill, prefill_tiles, read_status, sparse_latent, spec_flat,
    status_string, verify, verify_auto_splits, verify_noalloc, verify_workspace_size,
    wait_selftest, verify_shared, verify_shared_auto_splits, verify_fp8, transpose_spec,
    prefill_bwd, plan_prefill_bwd, prefill_bwd_tiles, verify_tree, verify_extend,
    PSA_OK, PSA_ERR_INVALID_ARG, PSA_ERR_UNSUPPORTED, PSA_ERR_WORKSPACE, PSA_ERR_CUDA,
    PSA_ERR_TIMEOUT, PSA_ERR_CAPACITY, PSA_ERR_BOUNDS, PSA_BF16, PSA_F32,
)
