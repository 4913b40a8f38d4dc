// Test helper (not part of libfp4): compares the quantizer's scale division
// (reciprocal + two FMA corrections, IEEE fallback) with CUDA's IEEE
// division __fdiv_rn for every finite bf16 dividend and a list of divisors.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../microscaling_fp4_quantization_mxfp4_b200/csrc/fp4_device.cuh"

__global__ void div_check_kernel(const float* scales, int n, unsigned long long* mismatches,
                                 unsigned long long* fallbacks) {
  const int s_idx = blockIdx.y;
  if (s_idx >= n) return;
  const float S = scales[s_idx];
  const float y = __frcp_rn(S);
  const bool usable = fp4dev::recip_usable(S);
  unsigned long long bad = 0, slow = 0;
  for (uint32_t b = blockIdx.x * blockDim.x + threadIdx.x; b < 65536u; b += gridDim.x * blockDim.x) {
    if (((b >> 7) & 0xFFu) == 0xFFu) continue;            // bf16 Inf/NaN
    const float x = __uint_as_float(b << 16);
    // the quantizer's per-block guard, applied to a one-element block
    const bool ok = usable && fp4dev::tiny_key(x) >= fp4dev::kTinyKeyMin && __fmul_rn(fabsf(x), y) < 0x1p64f;
    float q = ok ? fp4dev::div_by_recip(x, S, y) : __fdiv_rn(x, S);
    if (!ok) ++slow;
    const float ref = __fdiv_rn(x, S);
    if (__float_as_uint(q) != __float_as_uint(ref)) ++bad;
  }
  if (bad) atomicAdd(mismatches, bad);
  if (slow) atomicAdd(fallbacks, slow);
}

extern "C" int div_check(const float* scales, int n, unsigned long long* mismatches, unsigned long long* fallbacks) {
  dim3 grid(64, n);
  div_check_kernel<<<grid, 256>>>(scales, n, mismatches, fallbacks);
  return (int)cudaDeviceSynchronize();
}
