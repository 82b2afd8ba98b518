"""Blockwise exact ("ring") attention forward for NVIDIA B200 (sm_100a).

The compute lives in ``libringattn.so`` (C ABI: ``include/ring_attn.h``);
this package is its thin ctypes binding.  The library is loaded on first use.
"""

from ._binding import (  # noqa: F401
    BF16,
    CONTIGUOUS,
    EXPORTS,
    F16,
    F32,
    RA_ERR_CUDA,
    RA_ERR_INVALID,
    RA_ERR_TIMEOUT,
    RA_ERR_UNSUPPORTED,
    RA_OK,
    STRIPED,
    RingAttnError,
    library_path,
    load_library,
    ring_attn_bwd,
    ring_attn_bwd_simt,
    ring_attn_func,
    ring_attn_func_host,
    ring_attn_fwd,
    ring_attn_fwd_fp8,
    ring_attn_fwd_host,
    ring_attn_fwd_host_workspace,
    ring_attn_fwd_noalloc,
    ring_attn_noalloc_status,
    ring_attn_fwd_step,
    ring_attn_gqa_fwd,
    ring_attn_fwd_simt,
    ring_attn_merge,
    ring_attn_qkvpacked_fwd,
    ring_attn_qkvpacked_func,
    ring_attn_schedule,
    ring_attn_status,
    ring_attn_test_withhold_q,
    ring_attn_test_dump_schedule,
    ring_attn_status_string,
    ring_attn_varlen_qkvpacked_func,
)
