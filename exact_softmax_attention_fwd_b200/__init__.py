"""Exact softmax attention forward for B200 (sm_100a).

The compute lives in the CUDA C-ABI library ``libattn_b200.so`` (declared in
``include/attn.h``); this package is its thin ctypes binding plus the seeded
workload generators.  Importing the package does not load the library; the
first call does, and raises if the library is missing or no GPU is present.
"""
from ._binding import (  # noqa: F401
    AttnError,
    attn_bwd,
    attn_bwd_block_sparse,
    attn_bwd_varlen,
    attn_bwd_varlen_workspace_size,
    attn_bwd_window,
    attn_bwd_workspace_size,
    attn_fwd_block_sparse,
    attn_decode_paged,
    attn_decode_paged_fp8,
    attn_decode_workspace_size,
    attn_fwd,
    attn_fwd_fp8,
    attn_fwd_masked,
    attn_fwd_host,
    attn_fwd_host_workspace_size,
    attn_fwd_paged,
    attn_fwd_paged_fp8,
    attn_fwd_paged_fp8_workspace_size,
    attn_fwd_varlen,
    attn_fwd_varlen_workspace_size,
    attn_fwd_window,
    attn_get_device_error,
    attn_strerror,
    library_path,
    load_library,
)
