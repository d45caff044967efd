"""B200-native S6 selective scan: the fused forward, its backward and the recurrent step.

The compute lives in libssscan.so (hand-written sm_100a CUDA, C ABI in
include/ss_scan.h); this package is its Python binding plus the seeded input
generator (``selective_state_space_ss_b200.inputs``).  The library is loaded
lazily on the first call, and a missing library raises: there is no CPU path.
"""
from ._native import (  # noqa: F401
    EXPORTED,
    SS_DEBUG_CLEAR,
    SS_DEBUG_FORCE_SEGMENTS,
    SS_DEBUG_FORCE_WORKERS,
    SS_DEBUG_SKIP_PUBLISH,
    SS_DEBUG_SPIN_LIMIT,
    SS_DEBUG_STEP_SIMPLE,
    SS_BF16,
    SS_ERR_BOUNDS,
    SS_ERR_CUDA,
    SS_ERR_INVALID_ARG,
    SS_ERR_TIMEOUT,
    SS_ERR_UNSUPPORTED,
    SS_F32,
    SS_NOALLOC_SCRATCH_BYTES,
    SS_OK,
    SSError,
    library_path,
    load_library,
    ss_debug_fwd_kernels,
    ss_debug_inject,
    ss_last_device_error,
    ss_scan_bwd,
    ss_scan_bwd_workspace_bytes,
    ss_scan_fwd,
    ss_scan_fwd_conv,
    ss_scan_fwd_from_state,
    ss_scan_fwd_noalloc,
    ss_scan_fwd_train,
    ss_scan_fwd_zoh,
    ss_scan_step,
    ss_scan_workspace_bytes,
    ss_status_string,
)
