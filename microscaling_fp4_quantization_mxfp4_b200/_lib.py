"""ctypes loader for libfp4.so and the prototypes of include/fp4.h."""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp4.so")

_i64, _u64, _int, _vp, _sz = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/fp4.h
PROTOTYPES = {
    "fp4_quantize": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _int, _u64, _vp, _vp, _vp, _vp, _int, _vp]),
    "fp4_quantize_shard": (_int, [_vp, _i64, _i64, _i64, _i64, _int, _int, _int, _int, _u64, _vp, _vp, _vp, _vp, _int,
                                  _vp]),
    "fp4_hadamard_quantize": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _int, _u64, _vp, _vp, _vp, _vp,
                                     _int, _int, _vp, _vp]),
    "fp4_quantize_dequantize": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _u64, _vp, _vp, _vp, _vp, _int, _vp,
                                       _int, _vp]),
    "fp4_quantize_2d": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _u64, _vp, _vp, _vp, _vp, _vp, _vp,
                               _int, _vp]),
    "fp4_quantize_mse": (_int, [_vp, _i64, _i64, _i64, _int, _int, _int, _u64, _int, _vp, _vp, _vp, _int, _vp]),
    "fp4_dequantize": (_int, [_vp, _vp, _vp, _i64, _i64, _int, _int, _int, _vp, _int, _vp]),
    "fp4_gemm": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _vp, _i64, _int, _vp]),
    "fp4_gemm_quantize": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _int, _int, _int, _int, _int, _u64,
                                 _vp, _vp, _vp, _int, _vp]),
    "fp4_amax": (_int, [_vp, _i64, _i64, _i64, _vp, _vp]),
    "fp4_amax_noalloc": (_int, [_vp, _i64, _i64, _i64, _vp, _vp]),
    "fp4_nv_tensor_scale": (_int, [_vp, _vp, _vp]),
    "fp4_codes_bytes": (_sz, [_i64, _i64]),
    "fp4_scales_bytes": (_sz, [_i64, _i64, _int, _int, _int]),
    "fp4_check_device_errors": (_int, [_vp]),
    "fp4_status_string": (ctypes.c_char_p, [_int]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load the in-tree library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libfp4.so not found at {LIB_PATH}; build it with "
                "`python -m microscaling_fp4_quantization_mxfp4_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
