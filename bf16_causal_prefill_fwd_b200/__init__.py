"""Causal prefill attention forward for NVIDIA B200 (sm_100a), BF16 and FP8 e4m3.

The compute lives in libb200attn.so (hand-written CUDA for sm_100a behind the
C ABI in include/b200attn.h); this package is its thin Python binding.
"""
from ._binding import (  # noqa: F401
    B200AttnError,
    LIB_PATH,
    attn_func,
    attn_fwd,
    attn_fwd_fused_q,
    attn_varlen_func,
    attn_varlen_fwd,
    check,
    load_library,
    quantize_fp8,
    quantize_kv_fp8,
    quantize_kv_workspace_bytes,
    quantize_qkv_fp8,
    quantize_qkv_workspace_bytes,
    quantize_workspace_bytes,
    selftest_wait_timeout,
    version,
)
