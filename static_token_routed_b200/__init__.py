"""L³ (Large Lookup Layer) forward pass for one NVIDIA B200 (sm_100a).

The layer of "L³: Large Lookup Layers" (Tseng & De Sa; kimjy99 review,
Method, eq. L³) computes, per token with hidden state x and ID t,

    y = W_mix [ LayerNorm(W_up (V_t^T softmax(K_t x))) ; x ]

where K_t, V_t are the d_t-row slices of the concatenated tables W_K, W_V.
The work runs in hand-written CUDA kernels behind the C ABI in include/l3.h
(libl3.so); this package is the thin ctypes binding with the same names.
There is no CPU fallback: calls fail loudly when libl3.so is missing.
"""
from ._binding import (  # noqa: F401
    EXPORTED,
    L3_BF16,
    L3_FP32,
    Dims,
    KernelTime,
    L3Error,
    Plan,
    PlanInfo,
    l3_forward,
    l3_forward_status,
    l3_backward,
    l3_check_bounded_wait,
    l3_last_error,
    l3_lzw_allocate,
    l3_lzw_allocate_device,
    l3_plan,
    l3_plan_destroy,
    l3_plan_export,
    l3_plan_info,
    l3_plan_staged,
    l3_stage_rows,
    l3_profile_enable,
    l3_profile_read,
    l3_sort_tokens_noalloc,
    L3_SORT_NOALLOC_MAX_TOKENS,
    library,
    make_dims,
)
