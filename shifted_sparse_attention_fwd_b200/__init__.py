"""S²-Attn (LongLoRA shifted sparse attention) forward and backward for B200 (sm_100a).

The computation runs in libs2attn.so (C ABI: include/s2attn.h); this package is its
Python binding. Importing it does not load the library; the first call does, and raises
if the library is missing.
"""
from ._lib import (  # noqa: F401
    S2AttnError,
    S2ATTN_OK,
    S2ATTN_ERR_INVALID_ARG,
    S2ATTN_ERR_UNSUPPORTED,
    S2ATTN_ERR_CUDA,
    S2ATTN_ERR_TIMEOUT,
    S2ATTN_FLAG_WRAP_OWN_GROUP,
    S2ATTN_FLAG_WRAP_FRONT_FIRST,
    S2ATTN_FLAG_PARTIAL_LAST_GROUP,
    SIGNATURES,
    LIB_PATH,
    lib,
    status_string,
    s2attn_fwd,
    s2attn_fwd_rope_q,
    s2attn_bwd,
    s2attn_bwd_workspace_size,
    s2attn_bwd_workspace_size_ex,
    DEFAULT_WORKSPACE_CAP,
    s2attn_bwd_preprocess,
    s2attn_bwd_dkdv,
    s2attn_bwd_dq,
    s2attn_bwd_dkdv_ds,
    s2attn_bwd_dq_ds,
    s2attn_bwd_noalloc,
    s2attn_get_device_error,
    s2attn_set_wait_timeout_ns,
    s2attn_selftest_wait_timeout,
    s2attn_rope_pi,
    rope_pi,
    fwd,
    bwd,
)
