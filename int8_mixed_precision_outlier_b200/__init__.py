"""LLM.int8() mixed-precision decomposition matmul for B200 (sm_100a).

The compute path is the C-ABI library libllmint8.so (include/llmint8.h); the
functions here are its Python binding.
"""
from .llmint8 import (  # noqa: F401
    GEMV_MAX_T, PATH_AUTO, PATH_GEMM, PATH_GEMV, Int8Linear, LLMInt8Error, alloc_workspace,
    check_matmul_shapes, header_functions, llmint8_detect_quantize, llmint8_int8_gemm_i32, llmint8_kernel_launches, llmint8_matmul, llmint8_matmul_debug,
    llmint8_matmul_decode_noalloc, llmint8_matmul_intermediates, llmint8_matmul_profile,
    llmint8_quantize_weight, llmint8_selftest_timeout, llmint8_set_wait_limit_ns,
    llmint8_status_string, llmint8_sync_status, llmint8_version, llmint8_workspace_bytes,
    load_library, llmint8_column_absmax, llmint8_smooth_factors, llmint8_smoothquant_quantize_weight,
    llmint8_smoothquant_matmul, llmint8_fp8_quantize_weight, llmint8_fp8_matmul, llmint8_outlier_store_build,
    llmint8_matmul_stored,
)
