// Test helper (not part of libfp4): compares the quantizer's scale division
// (reciprocal + two FMA corrections, IEEE fallback) with CUDA's IEEE
// division __fdiv_rn for every finite bf16 dividend and a list of divisors,
// one element at a time (div_by_recip) and in 16-element blocks on packed
// pairs (nv_divide_block2: bit-identical quotients under the stochastic-rounding test,
// round-to-nearest codes under the round-to-nearest one).
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

__device__ __forceinline__ uint32_t rtn_code(float q) {
  uint32_t c;
  asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %1;\n\tcvt.u32.u8 %0, b;\n\t}" : "=r"(c) : "f"(q));
  return c & 0xFu;
}

// Blocks of 16 bf16 dividends: thread t takes patterns (t * 16 + i * stride) mod 2^16, i < 16
// (stride 1: neighbours of one magnitude; a large odd stride: tiny and large elements mixed).
// Quotients of elements with |x| >= 2^-103 (or 0) must equal IEEE division bit for bit; smaller
// ones must give the same round-to-nearest E2M1 code (RND = 0), or, under the stochastic-rounding
// test (RND = 1, which sends blocks with such elements to IEEE division), be equal too.
template <int RND>
__global__ void div_check_pair_kernel(const float* scales, int n, uint32_t stride, unsigned long long* mismatches,
                                      unsigned long long* fallbacks) {
  const int s_idx = blockIdx.y;
  if (s_idx >= n) return;
  const float S = scales[s_idx];
  const float2 sy = make_float2(S, fp4dev::recip_usable(S) ? __frcp_rn(S) : 0.0f);
  unsigned long long bad = 0, slow = 0;
  for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < 4096u; t += gridDim.x * blockDim.x) {
    float x[16], q[16];
    float am = 0.0f;
    bool finite = true;
    for (int i = 0; i < 16; ++i) {
      const uint32_t b = (t * 16u + (uint32_t)i * stride) & 0xFFFFu;
      finite = finite && ((b >> 7) & 0xFFu) != 0xFFu;
      x[i] = __uint_as_float(b << 16);
      q[i] = x[i];
      am = fmaxf(am, fabsf(x[i]));
    }
    if (!finite) continue;
    if (!fp4dev::nv_fast_division<RND, 16>(x, am, sy.x, sy.y)) ++slow;
    fp4dev::nv_divide_block2<RND, 16>(q, am, sy);
    for (int i = 0; i < 16; ++i) {
      const float ref = __fdiv_rn(x[i], S);
      const bool exact = RND == 1 || x[i] == 0.0f || fabsf(x[i]) >= 0x1p-103f;
      if (exact ? __float_as_uint(q[i]) != __float_as_uint(ref) : rtn_code(q[i]) != rtn_code(ref)) ++bad;
    }
  }
  if (bad) atomicAdd(mismatches, bad);
  if (slow) atomicAdd(fallbacks, slow);
}

extern "C" int div_check_pair(const float* scales, int n, unsigned stride, int rnd, unsigned long long* mismatches,
                              unsigned long long* fallbacks) {
  dim3 grid(16, n);
  if (rnd) {
    div_check_pair_kernel<1><<<grid, 256>>>(scales, n, stride, mismatches, fallbacks);
  } else {
    div_check_pair_kernel<0><<<grid, 256>>>(scales, n, stride, mismatches, fallbacks);
  }
  return (int)cudaDeviceSynchronize();
}

extern "C" int div_check(const float* scales, int n, unsigned long long* mismatches, unsigned long long* fallbacks) {
  dim3 grid(64, n);
  div_check_kernel<<<grid, 256>>>(scales, n, mismatches, fallbacks);
  return (int)cudaDeviceSynchronize();
}
