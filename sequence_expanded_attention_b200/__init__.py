"""sequence_expanded_attention_b200: B200-native (sm_100a) Hidden Decoding hot path.

The library is ``libhd.so`` (C ABI, declared in ``include/hd.h``): the n-table
embedding expansion, Stream-Factorized Attention prefill (within-stream and
cross-stream) and SFA decode over the retained expanded KV cache.  This package
is a thin ctypes binding over it; every step of the path runs in the CUDA
kernels.  Importing the package does not load the library; the first call does,
and raises if it is missing.
"""
from .binding import (  # noqa: F401
    SFA_WITHIN,
    SFA_CROSS,
    SFA_TRANSIENT,
    HD_DEV_ID_RANGE,
    HD_DEV_TIMEOUT,
    HD_DEV_BAD_LENGTH,
    HD_DEV_PAGE_RANGE,
    HdError,
    hd_expand_embed,
    hd_expand_embed_backward,
    hd_final_stream_rows,
    sfa_prefill_fwd,
    sfa_decode_fwd,
    sfa_decode_workspace_bytes,
    sfa_prefill_window_fwd,
    sfa_prefill_chunk_fwd,
    sfa_prefill_chunk_paged_fwd,
    sfa_prefill_bwd,
    sfa_prefill_bwd_workspace_bytes,
    sfa_decode_window_fwd,
    sfa_decode_window_workspace_bytes,
    sfa_decode_paged_fwd,
    sfa_decode_paged_workspace_bytes,
    library_path,
    load_library,
)
