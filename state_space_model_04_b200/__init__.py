"""B200-native (sm_100a) Mamba-2 SSD hot path: chunked prefill and O(1) cached decode.

The compute lives in libssd_b200.so (hand-written CUDA for sm_100a, C ABI in
include/ssd.h); this package is its thin Python binding.  Build it in-tree with
``python -m state_space_model_04_b200.build``.
"""
from .ssd import (  # noqa: F401
    SSD_ACT_NONE,
    SSD_ACT_SILU,
    SSD_BF16,
    SSD_F32,
    DecodePlan,
    SSDError,
    debug_decay_precision,
    debug_force_fma_prefill,
    debug_force_prefill_segments,
    debug_force_prefill_split,
    debug_starve_next_prefill,
    decode_loop,
    decode_step,
    decode_step_noalloc,
    decode_workspace_size,
    last_error,
    launch_count,
    lib,
    profile_begin,
    profile_end,
    prefill,
    prefill_check,
    prefill_context_scan,
    prefill_local_state,
    prefill_segments,
    prefill_whole_units,
    prefill_workspace_size,
    status_string,
)
