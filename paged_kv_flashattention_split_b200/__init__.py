"""B200-native paged-KV FlashAttention: decode, split-KV merge, causal extend, 8-bit Sage decode.

The compute lives in ``libpagedattn.so`` (hand-written CUDA for sm_100a, C ABI
in ``include/pagedattn.h``); this package is its thin Python binding, with the
same entry-point names, plus the in-tree build step.  PyTorch is used only for
device memory and streams.
"""
from ._binding import (  # noqa: F401
    EXPORTED,
    LIB_PATH,
    PA_ERR_ARCH,
    PA_ERR_CUDA,
    PA_ERR_DEVICE_INDEX,
    PA_ERR_INVALID,
    PA_ERR_UNSUPPORTED,
    PA_ERR_WORKSPACE,
    PA_MODE_DECODE,
    PA_MODE_EXTEND,
    PA_MODE_SAGE_DECODE,
    PA_MODE_SAGE_SPARSE,
    PA_OK,
    PagedAttnError,
    attn_debug_gather,
    attn_decode_paged,
    attn_decode_paged_fp8,
    attn_decode_paged_noalloc,
    attn_decode_paged_sage,
    attn_extend_paged,
    attn_extend_paged_sage,
    attn_kv_store,
    attn_kv_store_sage,
    attn_plan,
    attn_plan_sage_sparse,
    lib,
    make_params,
    pa_plan_params,
    pa_noalloc_read_device_error,
    pa_plan_workspace_size,
    pa_read_device_error,
    pa_version,
    status_string,
)
