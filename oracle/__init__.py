"""CPU oracle for microscaling FP4 quantization and the block-scaled FP4 GEMM.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) may import, call or link anything here; only `tests/`,
`__graft_entry__.smoke()` and the `cpu_baseline` / `--impl reference` legs of
`bench.py` use it.  It shares no code, tables or constants with the CUDA
sources: every number here is written out from the format definitions.

The oracle is deliberately plain and slow: NumPy, fp32 where the method's
arithmetic is fp32 (every operation correctly rounded, in the order written),
fp64 for the Hadamard rotation and the GEMM reference.  Sources, by page and
section:

* "FP4 All the Way: Fully Quantized Training of LLMs", Abstract: FP4 (E2M1)
  for weights, activations and gradients; NVFP4 = blocks of 16 E2M1 values
  sharing an E4M3 scale; round-to-nearest in the forward pass, stochastic
  rounding in the backward and update passes; block size, scale format and
  rounding are the design choices.
* "Bridging the Gap Between Promise and Performance for Microscaling FP4
  Quantization", Abstract: MXFP4 (power-of-two scales) and NVFP4; block-wise
  Hadamard transforms, fused into the weights and computed online for the
  activations; FP4 GEMM kernels on B200.  Its summary post (section 3 of the
  MR-GPTQ list): block-diagonal Hadamard rotations of the activations.
* "Oscillation-Reduced MXFP4 Training for Vision Transformers", Abstract: the
  MX format's fine-grained per-group scaling, supported by Blackwell.

The pages fix no bit-level encodings; where they are silent the oracle takes
the plainest reading (OCP MX v1.0 E2M1/E8M0/E4M3 conventions, Philox4x32-10 of
Salmon et al. SC'11, Sylvester Hadamard) and each module says which.

Modules: `formats` (E2M1/E4M3/E8M0), `philox`, `quantize` (MX/NV, RTN/SR,
axis 0/1, packing, dequantize; fmt "nvfp4_4o6" via `four_over_six`),
`quantize2d` (square-tile 2-D blocks), `mse_grid` (MSE-searched NVFP4 scales,
fmt "mxfp4_gs": MXFP4 with the MSE-fitted clip threshold),
`hadamard`, `layout` (tensor-core scale-factor layout), `gemm` (fp64 reference
and error bound).
"""
from .formats import (E2M1_GRID, e2m1_decode, e2m1_rtn, e2m1_sr, e4m3_decode, e4m3_rne_sat,
                      mx_scale_exponent)
from .philox import philox4x32_10, philox_words
from .hadamard import sylvester, block_hadamard
from .quantize import quantize, quantize_values, dequantize, pack_nibbles, unpack_nibbles, nv_tensor_scale
from .layout import sf_to_mma, sf_from_mma, sf_mma_bytes
from .gemm import gemm_ref, gemm_ref_rows, gemm_ref_cols, deq_for_gemm
from .quantize2d import quantize_2d
from .mse_grid import quantize_mse

__all__ = [
    "E2M1_GRID", "e2m1_decode", "e2m1_rtn", "e2m1_sr", "e4m3_decode", "e4m3_rne_sat",
    "mx_scale_exponent", "philox4x32_10", "philox_words", "sylvester", "block_hadamard",
    "quantize", "quantize_values", "dequantize", "pack_nibbles", "unpack_nibbles", "nv_tensor_scale",
    "sf_to_mma", "sf_from_mma", "sf_mma_bytes", "gemm_ref", "gemm_ref_rows", "gemm_ref_cols",
    "deq_for_gemm", "quantize_2d",
]
