"""Paged KV cache and paged-decode attention for NVIDIA B200 (sm_100a).

The C library ``libpa.so`` (kernels + host block manager, interface in
``include/pa.h``) does the work; this package is its ctypes binding
(``_lib``), a build script (``build``) and a runner that drives one decode
step of a workload through the library (``runner``).
"""

from ._lib import (  # noqa: F401
    BLOCK_SIZE,
    BlockManager,
    PAError,
    PA_BF16,
    PA_DEVERR_BLOCK_RANGE,
    PA_DEVERR_CONTEXT_RANGE,
    PA_DEVERR_GROUP,
    PA_DEVERR_SLOT_RANGE,
    PA_DEVERR_WAIT_TIMEOUT,
    PA_F16,
    PA_FP8_E4M3,
    PA_PREEMPT_RECOMPUTE,
    PA_PREEMPT_SWAP,
    PA_SCHED_CASCADE_AUTO,
    PA_SCHED_CASCADE_OFF,
    PA_SCHED_CASCADE_ON,
    PrefixGroups,
    Scheduler,
    cascade_workspace,
    decode_workspace,
    last_error,
    lib,
    pa_cascade_order,
    pa_copy_blocks,
    pa_longest_first_order,
    pa_paged_decode,
    pa_paged_decode_cascade,
    pa_paged_decode_cascade_workspace_size,
    pa_paged_decode_fp8,
    pa_paged_decode_noalloc,
    pa_paged_decode_plan,
    pa_paged_decode_cascade_plan,
    pa_paged_decode_workspace_size,
    pa_reshape_and_cache,
    pa_reshape_and_cache_fp8,
    pa_swap_blocks,
)
