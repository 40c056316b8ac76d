"""B200-native ARL2 hybrid attention layer.

A thin ctypes binding of ``libhyb_attn.so`` (built from ``csrc/`` by
``gated_delta_linear_b200/build.py``).  The functions carry the C names of
``include/hyb_attn.h`` and only marshal arguments: every step of the layer
runs in the library's CUDA kernels.  Importing this package fails loudly when
the library has not been built.
"""

from ._binding import (  # noqa: F401
    HYB_OK,
    HYB_WARN_NONFINITE,
    HYB_ERR_INVALID,
    HYB_ERR_UNSUPPORTED,
    HYB_ERR_ALIGN,
    HYB_ERR_WORKSPACE,
    HYB_ERR_CUDA,
    HYB_ERR_TIMEOUT,
    HYB_BF16,
    HYB_FP32,
    HybAttnDesc,
    HybAttnError,
    lib,
    library_path,
    make_desc,
    hyb_attn_workspace_bytes,
    hyb_attn_forward,
    hyb_attn_forward_branches,
    hyb_attn_forward_next,
    hyb_attn_forward_noalloc,
    HYB_NOALLOC_SCRATCH_BYTES,
    hyb_attn_get_device_status,
    hyb_attn_status_string,
    hyb_kvcache_attn_forward,
    hyb_attn_forward_mixed,
    HybridAttention,
    TokenLevelAttention,
    hyb_attn_forward_token_level,
    hyb_attn_forward_frames,
    HybTraParams,
    hyb_tra_forward,
    hyb_tra_workspace_bytes,
    hyb_attn_frames_workspace_bytes,
    hyb_attn_token_level_workspace_bytes,
    KVCacheAttention,
    HybAttnTiming,
    HYB_NUM_KERNELS,
    hyb_attn_set_fault_test,
    hyb_attn_noalloc_device_status,
    hyb_attn_timing_begin,
    hyb_attn_timing_end,
    hyb_attn_kernel_name,
)
