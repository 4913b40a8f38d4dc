"""Thin Python binding of libfp4 (include/fp4.h), one function per C entry point.

Argument marshalling only: tensors are checked for device, dtype and layout,
output buffers are allocated with PyTorch when the caller gives none, and the
raw pointers plus the current CUDA stream go to the C ABI.  Every step of the
computation runs in the library's CUDA kernels; there is no CPU path, and
every call raises if libfp4.so is missing or a tensor is not on a GPU.
"""
from __future__ import annotations

from typing import NamedTuple, Optional

import torch

from . import _lib

MXFP4, NVFP4, NVFP4_4O6, MXFP4_GS = 0, 1, 2, 3
RTN, SR = 0, 1
SF_ROWMAJOR, SF_MMA = 0, 1
OUT_F32, OUT_BF16 = 0, 1

_FMT = {"mxfp4": MXFP4, "nvfp4": NVFP4, "nvfp4_4o6": NVFP4_4O6, "mxfp4_gs": MXFP4_GS,
        MXFP4: MXFP4, NVFP4: NVFP4, NVFP4_4O6: NVFP4_4O6, MXFP4_GS: MXFP4_GS}
_RND = {"rtn": RTN, "sr": SR, RTN: RTN, SR: SR}
_SF = {"rowmajor": SF_ROWMAJOR, "mma": SF_MMA, SF_ROWMAJOR: SF_ROWMAJOR, SF_MMA: SF_MMA}
_OUT = {"f32": OUT_F32, "bf16": OUT_BF16, torch.float32: OUT_F32, torch.bfloat16: OUT_BF16,
        OUT_F32: OUT_F32, OUT_BF16: OUT_BF16}
BLOCK = {MXFP4: 32, NVFP4: 16, NVFP4_4O6: 16, MXFP4_GS: 32}


class Fp4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.load().fp4_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


class Fp4Quantized(NamedTuple):
    codes: torch.Tensor          # uint8 [out_rows, L/2]
    scales: torch.Tensor         # uint8, row-major [out_rows, L/block] or flat tensor-core layout
    tensor_scale: Optional[torch.Tensor]   # fp32 [1] (NVFP4) or None


def _check(status: int, where: str) -> None:
    if status != 0:
        raise Fp4Error(status, where)


def _stream(stream) -> int:
    """cudaStream_t of `stream`, or of the current device's current stream (read as a raw handle,
    without building a Stream object)."""
    if stream is not None:
        return stream.cuda_stream
    return torch._C._cuda_getCurrentRawStream(torch._C._cuda_getDevice())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need_cuda(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libfp4 has no CPU path)")


def _bf16_matrix(x: torch.Tensor, name: str = "x") -> None:
    _need_cuda(x, name)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D bf16 CUDA tensor with unit column stride")


def fp4_codes_bytes(rows: int, cols: int) -> int:
    """Bytes of packed codes for a [rows, cols] tensor (two E2M1 codes per byte); 0 for an empty
    or odd-sized tensor."""
    return _lib.load().fp4_codes_bytes(rows, cols)


def fp4_scales_bytes(rows: int, cols: int, block: int, axis: int, sf_layout="rowmajor") -> int:
    """Bytes of block scales for a [rows, cols] tensor quantized along `axis` in `block`-element
    blocks: one byte per block row-major, or the tensor-core layout padded to 128 rows x 4 block
    columns ("mma"); 0 for an invalid shape."""
    return _lib.load().fp4_scales_bytes(rows, cols, block, axis, _SF[sf_layout])


def fp4_status_string(status: int) -> str:
    """Short message for an fp4_status code (e.g. "invalid argument" for FP4_ERR_ARG)."""
    return _lib.load().fp4_status_string(status).decode()


def fp4_check_device_errors(stream=None) -> None:
    """Synchronize and raise if a bounded device wait expired since the last check."""
    _check(_lib.load().fp4_check_device_errors(_stream(stream)), "fp4_check_device_errors")


def _alloc_quant_outputs(x, fmt, axis, sf, codes, scales, ts_out):
    rows, cols = x.shape
    orows, qlen = (rows, cols) if axis == 1 else (cols, rows)
    if codes is None:
        codes = torch.empty((orows, qlen // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        nbytes = fp4_scales_bytes(rows, cols, BLOCK[fmt], axis, sf)
        if nbytes == 0:
            raise ValueError("shape not quantizable with this block size along this axis")
        shape = (orows, qlen // BLOCK[fmt]) if sf == SF_ROWMAJOR else (nbytes,)
        scales = torch.empty(shape, dtype=torch.uint8, device=x.device)
    if fmt in (NVFP4, NVFP4_4O6) and ts_out is None:
        ts_out = torch.empty((1,), dtype=torch.float32, device=x.device)
    return codes, scales, ts_out


def fp4_quantize(x: torch.Tensor, fmt="mxfp4", axis: int = 1, rnd="rtn", seed: int = 0,
                 tensor_scale_in: Optional[torch.Tensor] = None, sf_layout="rowmajor", *,
                 codes=None, scales=None, tensor_scale_out=None, first_row: int = 0, stream=None) -> Fp4Quantized:
    """Block-scaled FP4 quantization of a bf16 matrix (see fp4_quantize in include/fp4.h).  With
    first_row > 0, x is a row shard of a larger tensor starting at that row (fp4_quantize_shard)."""
    _bf16_matrix(x)
    f, r, sf = _FMT[fmt], _RND[rnd], _SF[sf_layout]
    codes, scales, ts_out = _alloc_quant_outputs(x, f, axis, sf, codes, scales, tensor_scale_out)
    lib = _lib.load()
    if first_row:
        st = lib.fp4_quantize_shard(
            x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), first_row, f, BLOCK[f], axis, r,
            seed & (2 ** 64 - 1), _ptr(tensor_scale_in), _ptr(ts_out), codes.data_ptr(), scales.data_ptr(), sf,
            _stream(stream))
        _check(st, "fp4_quantize_shard")
    else:
        st = lib.fp4_quantize(
            x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), f, BLOCK[f], axis, r, seed & (2 ** 64 - 1),
            _ptr(tensor_scale_in), _ptr(ts_out), codes.data_ptr(), scales.data_ptr(), sf, _stream(stream))
        _check(st, "fp4_quantize")
    return Fp4Quantized(codes, scales, ts_out if f in (NVFP4, NVFP4_4O6) else None)


def fp4_hadamard_quantize(x: torch.Tensor, had_block: int, fmt="mxfp4", axis: int = 1, rnd="rtn",
                          seed: int = 0, tensor_scale_in=None, sf_layout="rowmajor", *, codes=None,
                          scales=None, tensor_scale_out=None, rotated_out=None, stream=None) -> Fp4Quantized:
    """Block-Hadamard rotation fused ahead of the quantizer (see include/fp4.h)."""
    _bf16_matrix(x)
    f, r, sf = _FMT[fmt], _RND[rnd], _SF[sf_layout]
    codes, scales, ts_out = _alloc_quant_outputs(x, f, axis, sf, codes, scales, tensor_scale_out)
    st = _lib.load().fp4_hadamard_quantize(
        x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), f, BLOCK[f], axis, r, seed & (2 ** 64 - 1),
        _ptr(tensor_scale_in), _ptr(ts_out), codes.data_ptr(), scales.data_ptr(), sf, had_block,
        _ptr(rotated_out), _stream(stream))
    _check(st, "fp4_hadamard_quantize")
    return Fp4Quantized(codes, scales, ts_out if f in (NVFP4, NVFP4_4O6) else None)


def fp4_quantize_dequantize(x: torch.Tensor, fmt="nvfp4", rnd="rtn", seed: int = 0,
                            tensor_scale_in: Optional[torch.Tensor] = None, sf_layout="rowmajor", out_dtype="f32", *,
                            codes=None, scales=None, tensor_scale_out=None, out=None, stream=None):
    """fp4_quantize along rows plus the dequantized values in the same launch (see include/fp4.h).
    Returns (Fp4Quantized, dequantized tensor)."""
    _bf16_matrix(x)
    f, r, sf, od = _FMT[fmt], _RND[rnd], _SF[sf_layout], _OUT[out_dtype]
    codes, scales, ts_out = _alloc_quant_outputs(x, f, 1, sf, codes, scales, tensor_scale_out)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float32 if od == OUT_F32 else torch.bfloat16, device=x.device)
    st = _lib.load().fp4_quantize_dequantize(
        x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), f, BLOCK[f], r, seed & (2 ** 64 - 1),
        _ptr(tensor_scale_in), _ptr(ts_out), codes.data_ptr(), scales.data_ptr(), sf, out.data_ptr(), od,
        _stream(stream))
    _check(st, "fp4_quantize_dequantize")
    return Fp4Quantized(codes, scales, ts_out if f in (NVFP4, NVFP4_4O6) else None), out


def fp4_quantize_2d(x: torch.Tensor, fmt="nvfp4", rnd="rtn", seed: int = 0,
                    tensor_scale_in: Optional[torch.Tensor] = None, sf_layout="rowmajor", transposed: bool = True,
                    *, codes=None, scales=None, codes_t=None, scales_t=None, tensor_scale_out=None,
                    stream=None):
    """Square-tile (2-D) quantization (see fp4_quantize_2d in include/fp4.h).  Returns
    (W along its rows, W^T along its rows or None) as Fp4Quantized, sharing one tensor scale."""
    _bf16_matrix(x)
    f, r, sf = _FMT[fmt], _RND[rnd], _SF[sf_layout]
    codes, scales, ts_out = _alloc_quant_outputs(x, f, 1, sf, codes, scales, tensor_scale_out)
    if transposed:
        codes_t, scales_t, _ = _alloc_quant_outputs(x, f, 0, sf, codes_t, scales_t, ts_out)
    else:
        codes_t = scales_t = None
    st = _lib.load().fp4_quantize_2d(
        x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), f, BLOCK[f], r, seed & (2 ** 64 - 1),
        _ptr(tensor_scale_in), _ptr(ts_out), codes.data_ptr(), scales.data_ptr(), _ptr(codes_t), _ptr(scales_t),
        sf, _stream(stream))
    _check(st, "fp4_quantize_2d")
    ts = ts_out if f == NVFP4 else None
    return Fp4Quantized(codes, scales, ts), (Fp4Quantized(codes_t, scales_t, ts) if transposed else None)


def fp4_quantize_mse(x: torch.Tensor, rnd="rtn", seed: int = 0, iters: int = 1, sf_layout="rowmajor", *,
                     codes=None, scales=None, tensor_scale_out=None, stream=None) -> Fp4Quantized:
    """NVFP4 quantization along rows with MSE-searched block and tensor scales (see fp4_quantize_mse in
    include/fp4.h); outputs are plain NVFP4."""
    _bf16_matrix(x)
    r, sf = _RND[rnd], _SF[sf_layout]
    codes, scales, ts_out = _alloc_quant_outputs(x, NVFP4, 1, sf, codes, scales, tensor_scale_out)
    st = _lib.load().fp4_quantize_mse(
        x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), NVFP4, 16, r, seed & (2 ** 64 - 1), iters,
        ts_out.data_ptr(), codes.data_ptr(), scales.data_ptr(), sf, _stream(stream))
    _check(st, "fp4_quantize_mse")
    return Fp4Quantized(codes, scales, ts_out)


def fp4_dequantize(codes: torch.Tensor, scales: torch.Tensor, tensor_scale=None, fmt="mxfp4",
                   sf_layout="rowmajor", out_dtype="f32", *, out=None, stream=None) -> torch.Tensor:
    """Codes + scales (+ tensor scale) back to fp32 or bf16 [rows, 2 * codes.shape[1]]."""
    _need_cuda(codes, "codes")
    f, sf, od = _FMT[fmt], _SF[sf_layout], _OUT[out_dtype]
    rows, cols = codes.shape[0], codes.shape[1] * 2
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32 if od == OUT_F32 else torch.bfloat16,
                          device=codes.device)
    st = _lib.load().fp4_dequantize(codes.data_ptr(), scales.data_ptr(), _ptr(tensor_scale), rows, cols, f,
                                    BLOCK[f], sf, out.data_ptr(), od, _stream(stream))
    _check(st, "fp4_dequantize")
    return out


def fp4_gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor,
             fmt="mxfp4", a_tensor_scale=None, b_tensor_scale=None, out_dtype="bf16", *, out=None,
             stream=None) -> torch.Tensor:
    """Y[M,N] = alpha * A . B^T on the FP4 tensor cores; scales in the tensor-core ("mma") layout."""
    for t, n in ((a_codes, "a_codes"), (b_codes, "b_codes"), (a_scales, "a_scales"), (b_scales, "b_scales")):
        _need_cuda(t, n)
    f, od = _FMT[fmt], _OUT[out_dtype]
    M, kb = a_codes.shape
    N, kb2 = b_codes.shape
    if kb != kb2:
        raise ValueError("A and B must have the same K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32 if od == OUT_F32 else torch.bfloat16, device=a_codes.device)
    st = _lib.load().fp4_gemm(a_codes.data_ptr(), a_scales.data_ptr(), _ptr(a_tensor_scale), b_codes.data_ptr(),
                              b_scales.data_ptr(), _ptr(b_tensor_scale), M, N, 2 * kb, f, BLOCK[f],
                              out.data_ptr(), out.stride(0), od, _stream(stream))
    _check(st, "fp4_gemm")
    return out


def fp4_gemm_quantize(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor,
                      fmt="mxfp4", a_tensor_scale=None, b_tensor_scale=None, out_fmt="mxfp4", rnd="rtn", seed: int = 0,
                      out_tensor_scale: Optional[torch.Tensor] = None, out_sf_layout="mma", *, codes=None, scales=None,
                      stream=None) -> Fp4Quantized:
    """Y = alpha * A . B^T quantized along its rows in the GEMM epilogue (see fp4_gemm_quantize in
    include/fp4.h): the next layer's FP4 operand, Y itself never written."""
    for t, n in ((a_codes, "a_codes"), (b_codes, "b_codes"), (a_scales, "a_scales"), (b_scales, "b_scales")):
        _need_cuda(t, n)
    f, of, r, sf = _FMT[fmt], _FMT[out_fmt], _RND[rnd], _SF[out_sf_layout]
    M, kb = a_codes.shape
    N, kb2 = b_codes.shape
    if kb != kb2:
        raise ValueError("A and B must have the same K")
    if codes is None:
        codes = torch.empty((M, N // 2), dtype=torch.uint8, device=a_codes.device)
    if scales is None:
        nbytes = fp4_scales_bytes(M, N, BLOCK[of], 1, sf)
        shape = (M, N // BLOCK[of]) if sf == SF_ROWMAJOR else (nbytes,)
        scales = torch.empty(shape, dtype=torch.uint8, device=a_codes.device)
    st = _lib.load().fp4_gemm_quantize(
        a_codes.data_ptr(), a_scales.data_ptr(), _ptr(a_tensor_scale), b_codes.data_ptr(), b_scales.data_ptr(),
        _ptr(b_tensor_scale), M, N, 2 * kb, f, BLOCK[f], of, BLOCK[of], r, seed & (2 ** 64 - 1),
        _ptr(out_tensor_scale), codes.data_ptr(), scales.data_ptr(), sf, _stream(stream))
    _check(st, "fp4_gemm_quantize")
    return Fp4Quantized(codes, scales, out_tensor_scale if of == NVFP4 else None)


def fp4_amax(x: torch.Tensor, *, out=None, stream=None) -> torch.Tensor:
    """max |x| of a bf16 matrix as a device fp32 [1]."""
    _bf16_matrix(x)
    if out is None:
        out = torch.empty((1,), dtype=torch.float32, device=x.device)
    _check(_lib.load().fp4_amax(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), out.data_ptr(),
                                _stream(stream)), "fp4_amax")
    return out


def fp4_nv_tensor_scale(amax: torch.Tensor, *, out=None, stream=None) -> torch.Tensor:
    """NVFP4 tensor scale amax / (6 * 448) (1.0 for amax == 0), computed on the device."""
    _need_cuda(amax, "amax")
    if out is None:
        out = torch.empty((1,), dtype=torch.float32, device=amax.device)
    _check(_lib.load().fp4_nv_tensor_scale(amax.data_ptr(), out.data_ptr(), _stream(stream)),
           "fp4_nv_tensor_scale")
    return out
