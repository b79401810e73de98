"""B200-native dynamic FP8 quantization (amax -> scale -> saturating RNE cast)
and the scaled FP8 GEMM it feeds.

The compute path is libhq.so (hand-written CUDA for sm_100a behind the C ABI
in include/hq.h); this package is its thin Python binding.
"""
from ._hq import (  # noqa: F401
    BF16, E4M3, E5M2, EXPORTED, F16, F32, LIB_PATH, PER_CHANNEL, PER_TENSOR, PER_TOKEN, DelayedTensor, HQError,
    check, hq_check_device_error, hq_dequantize_fp8_blockwise, hq_gemm_a8w8, hq_gemm_a8w8_blockq, hq_gemm_a8w8_ex,
    hq_gemm_blockscaled,
    hq_grad_bias, hq_grad_bias_workspace_bytes,
    hq_granularity_name, hq_grouped_gemm_a8w8, hq_grouped_gemm_bf16, hq_linear_blockwise,
    hq_quantize_e5m2_stochastic, hq_quantize_fp8, hq_quantize_fp8_blockwise, hq_quantize_fp8_delayed_batch,
    hq_quantize_fp8_noalloc, hq_quantize_fp8_transpose, hq_quantize_workspace_bytes, hq_scale_count,
    hq_scale_pair_name, hq_version, lib,
)
