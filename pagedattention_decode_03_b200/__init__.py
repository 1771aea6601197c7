"""Paged single-query decode attention for NVIDIA B200 (sm_100a).

The work happens in ``libpa.so`` (C ABI in ``include/pa.h``): a host-side
block manager (free list, block tables, reference counts, copy-on-write),
the append kernel that writes new K/V rows into their cache slots, and the
decode-attention kernels (tensor-core and CUDA-core paths, split-KV with a
log-sum-exp reduction, FP8-E4M3 KV).  This package is a thin ctypes
binding with the same names; importing it does not load the library, the
first call does, and raises if it has not been built.
"""
from .binding import (  # noqa: F401
    DTYPES,
    EXPORTS,
    LIB_PATH,
    PA_DEVERR_BAD_BLOCK,
    PA_DEVERR_BAD_LEN,
    PA_DEVERR_TIMEOUT,
    PA_ERR_CUDA,
    PA_ERR_DEVICE_CHECK,
    PA_ERR_INVALID_ARG,
    PA_ERR_NO_BLOCKS,
    PA_ERR_NO_SEQ,
    PA_ERR_SEQ_EXISTS,
    PA_ERR_SHARED_BLOCK,
    PA_OK,
    PAError,
    Pool,
    lib,
    pa_alloc_blocks,
    pa_alloc_blocks_n,
    pa_alloc_blocks_prefix,
    pa_append_kv,
    pa_check_device_errors,
    pa_debug_fail_after,
    pa_decode_attention,
    pa_decode_attention_append,
    pa_decode_attention_noalloc,
    pa_fork_cow,
    pa_free,
    pa_get_cached_blocks,
    pa_get_cow_log,
    pa_get_free_list,
    pa_get_refcounts,
    pa_last_decode_plan,
    pa_plan_siblings,
    pa_prefix_match,
    pa_prefix_register,
    pa_get_seq,
    pa_last_error,
    pa_launch_count,
    pa_pool_create,
    pa_pool_destroy,
    pa_status_string,
    pa_swap_bytes,
    pa_swap_in,
    pa_swap_out,
    pa_workspace_size,
)
