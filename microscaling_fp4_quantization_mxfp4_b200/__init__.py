"""B200-native (sm_100a) microscaling FP4 quantization and block-scaled FP4 GEMM.

The compute lives in libfp4.so (hand-written CUDA: quantize / Hadamard-quantize /
dequantize / tensor-amax kernels and a tcgen05 block-scaled GEMM); this package
is the thin Python binding plus the multi-rank helper.  See include/fp4.h for
the C ABI.
"""
from .binding import (BLOCK, MXFP4, MXFP4_GS, NVFP4, NVFP4_4O6, OUT_BF16, OUT_F32, RTN, SF_MMA, SF_ROWMAJOR, SR,
                      Fp4Error, Fp4Quantized, fp4_amax, fp4_check_device_errors, fp4_codes_bytes, fp4_dequantize,
                      fp4_gemm, fp4_gemm_quantize, fp4_hadamard_quantize, fp4_nv_tensor_scale, fp4_quantize, fp4_quantize_2d,
                      fp4_quantize_dequantize,
                      fp4_quantize_mse, fp4_scales_bytes, fp4_status_string)

__all__ = [
    "BLOCK", "MXFP4", "MXFP4_GS", "NVFP4", "NVFP4_4O6", "OUT_BF16", "OUT_F32", "RTN", "SF_MMA", "SF_ROWMAJOR", "SR",
    "Fp4Error", "Fp4Quantized", "fp4_amax", "fp4_check_device_errors", "fp4_codes_bytes", "fp4_dequantize", "fp4_gemm", "fp4_gemm_quantize",
    "fp4_hadamard_quantize", "fp4_nv_tensor_scale", "fp4_quantize", "fp4_quantize_2d", "fp4_quantize_dequantize", "fp4_quantize_mse",
    "fp4_scales_bytes", "fp4_status_string",
]
