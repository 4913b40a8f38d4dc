// NVFP4 quantization with MSE-searched scales (sm_100a).
//
// The summary post of "Bridging the Gap Between Promise and Performance for Microscaling FP4
// Quantization" (its MR-GPTQ list, item 1) makes the FP4 grid MSE-effective by optimizing it
// alternately at the scale of each block and of the tensor.  Here:
//   * block step (tensor scale s fixed): each 16-element block takes, among the eight E4M3 bytes
//     below and above its standard byte b6 (and b6 itself), the one whose round-to-nearest result
//     has the least squared error -- error in fp64, terms added in element order, ties to the
//     byte met first in the order b6, b6-1, b6+1, b6-2, ...;
//   * tensor step: s is replaced by the best of s * (1 + k/64), k = -8..8, each scored after its
//     own block step by Q = sum over blocks of floor(err_b * 2^P), P = 80 - 2 floor(log2 amax):
//     integers below 2^87 whose sum is exact in any order, so the choice does not depend on how
//     the reduction is parallelised.
// The schedule is s = amax / 2688, `iters` tensor steps, then a block step whose bytes quantize
// the codes (RTN or Philox SR).  One thread owns one block.  Each candidate byte is first scored
// in fp32 from quotients by the reciprocal (a multiply instead of a correctly rounded division);
// only candidates that the screen's error bound cannot rule out are scored exactly (exact
// quotients, fp64 errors), so the fp64 argmin is found without evaluating every candidate in fp64.
// Inputs are finite bf16.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fp4_device.cuh"
#include "fp4_internal.h"

using namespace fp4dev;

namespace fp4lib {
namespace {

constexpr int kWindow = 8;                    // block step: bytes b6 - 8 .. b6 + 8
constexpr int kCands = 2 * kWindow + 1;
constexpr int kTensorCands = 17;              // tensor step: s * (1 + k/64), k = -8..8
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Offset of candidate j in tie-break order: 0, -1, +1, -2, +2, ...
__device__ __forceinline__ int cand_offset(int j) { return (j & 1) ? -((j + 1) >> 1) : (j >> 1); }

// Tensor-step multipliers 1 + k/64, k = -8..8 (exact in fp32), and the candidate scales.
__device__ __forceinline__ float step_scale(float s, int k) {
  return __fmul_rn(s, 1.0f + (float)(k - kTensorCands / 2) * 0.015625f);
}

struct MseParams {
  const uint16_t* x;     // bf16 [rows, cols] with row stride ld
  int64_t ld;
  uint32_t nblocks;      // rows * cols / 16
  uint32_t bpr;          // blocks per row
  uint32_t g4;           // padded k-groups / 4 (tensor-core scale layout)
  const float* amax;     // tensor amax
  float* s_t;            // tensor scale: read (unless from_amax) and written
  int from_amax;         // start from s = amax / 2688 (1 for an all-zero tensor)
  unsigned long long* partials;   // tensor step: [gridDim.x][kTensorCands][2]
  unsigned* ticket;      // tensor step: CTA completion counter (self-resetting)
  uint8_t* codes;        // [rows, cols / 2]
  uint8_t* scales;       // row-major [rows, cols / 16] or the tensor-core layout
  int sf_mma;
  PhiloxKeys keys;
};

__device__ __forceinline__ float start_scale(const MseParams& p) {
  if (!p.from_amax) return *p.s_t;
  const float a = *p.amax;
  return a == 0.0f ? 1.0f : __fdiv_rn(a, 2688.0f);
}

__device__ __forceinline__ void load_block(const MseParams& p, uint32_t blk, float (&x)[16], float& am) {
  const uint32_t row = blk / p.bpr, g = blk - row * p.bpr;
  const uint4* src = reinterpret_cast<const uint4*>(p.x + (int64_t)row * p.ld + 16 * g);
  const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
  float a[8], b[8];
  unpack8(v0, a);
  unpack8(v1, b);
  am = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[i] = a[i];
    x[8 + i] = b[i];
    am = fmaxf(am, fmaxf(fabsf(a[i]), fabsf(b[i])));
  }
}

// RTN grid points (signed E2M1 values) of two scaled values.
__device__ __forceinline__ float2 e2m1_rtn_value2(float q0, float q1) {
  uint32_t h;
  asm("{\n\t.reg .b8 c;\n\tcvt.rn.satfinite.e2m1x2.f32 c, %2, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
      : "=r"(h)
      : "f"(q0), "f"(q1));
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// fp32 screen of the byte with divisor sy.x = S and sy.y = RN(1/S): quotients q = x * RN(1/S) (not
// correctly rounded), their round-to-nearest grid points G(q), and S^2 * sum (q - G(q))^2.  The
// squared distance to the nearest grid point is 1-Lipschitz in q, so against the exact error each
// element is off by at most ~16.5u x^2 (u = 2^-24; q within 2u of x/S, the method's own quotient
// and dequantized value within 6u), and the fp32 sums add 20u relatively.
__device__ __forceinline__ float screen32(const float (&x)[16], float2 sy) {
  float f = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float q0 = __fmul_rn(x[i], sy.y), q1 = __fmul_rn(x[i + 1], sy.y);
    const float2 g = e2m1_rtn_value2(q0, q1);
    float e = __fsub_rn(q0, g.x);
    f = __fmaf_rn(e, e, f);
    e = __fsub_rn(q1, g.y);
    f = __fmaf_rn(e, e, f);
  }
  return __fmul_rn(f, __fmul_rn(sy.x, sy.x));
}

// Exact error of byte b (0: the block dequantizes to 0): fp64 terms in element order.
__device__ __forceinline__ double score64(const float (&x)[16], float am, uint32_t b, float s, const float2* tab) {
  double acc = 0.0;
  if (b == 0u) {
#pragma unroll
    for (int i = 0; i < 16; ++i) acc = __fma_rn((double)x[i], (double)x[i], acc);
    return acc;
  }
  float q[16];
  nv_divide_block<0, 16>(x, am, tab[b], q);
  const __half2 g = __float2half2_rn(e4m3_value(b));
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float2 d = nv_rtn_dequant2(q[i], q[i + 1], g, s);
    double e = __dsub_rn((double)x[i], (double)d.x);
    acc = __fma_rn(e, e, acc);
    e = __dsub_rn((double)x[i + 1], (double)d.y);
    acc = __fma_rn(e, e, acc);
  }
  return acc;
}

// Block step for one block under tensor scale s (tab: its (S, 1/S) table).  Returns the byte;
// with want_err, *err receives its exact error.
__device__ __forceinline__ uint32_t block_byte(const float (&x)[16], float am, float s, float y_s, bool s_ok,
                                               const float2* tab, bool want_err, double* err) {
  const int b6 = (int)e4m3_rn_sat(nv_scale_arg(am, s, y_s, s_ok));
  if (b6 == 0) {
    if (want_err) *err = score64(x, am, 0u, s, tab);
    return 0u;
  }
  // fp32 screen of every candidate (NaN marks a byte whose quotients the screen cannot bound:
  // unusable reciprocal or huge quotients; it always goes to the exact stage)
  float x2 = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) x2 = __fmaf_rn(x[i], x[i], x2);
  float f[kCands];
  float m = __int_as_float(0x7F800000);
#pragma unroll
  for (int j = 0; j < kCands; ++j) {
    const int b = b6 + cand_offset(j);
    float v = __int_as_float(0x7F800000);
    if (b >= 1 && b <= 126) {
      const float2 sy = tab[b];
      v = (sy.y != 0.0f && __fmul_rn(am, sy.y) < 0x1p64f) ? screen32(x, sy) : __int_as_float(0x7FC00000);
    }
    f[j] = v;
    m = fminf(m, v);
  }
  // candidates whose exact error may be the least: a screen score exceeds the best one by more
  // than 2^-16 (sum x^2 + both scores) + 2^-120 -- eight times the two scores' error bounds --
  // only if its exact error is larger too; an infinite best score keeps every candidate
  int count = 0, first = 0;
#pragma unroll
  for (int j = kCands - 1; j >= 0; --j) {
    const int b = b6 + cand_offset(j);
    const float tol = __fmaf_rn(__fadd_rn(x2, __fadd_rn(m, f[j])), 0x1p-16f, 0x1p-120f);
    if (b >= 1 && b <= 126 && !(__fsub_rn(f[j], m) > tol)) {
      ++count;
      first = j;
    }
  }
  if (count == 1) {
    const uint32_t b = (uint32_t)(b6 + cand_offset(first));
    if (want_err) *err = score64(x, am, b, s, tab);
    return b;
  }
  // close call (or no finite score): exact errors of the contenders, in tie-break order
  uint32_t best = 0u;
  double be = 0.0;
  bool have = false;
  for (int j = 0; j < kCands; ++j) {
    const int b = b6 + cand_offset(j);
    if (b < 1 || b > 126) continue;
    float fj = 0.0f;
#pragma unroll
    for (int t = 0; t < kCands; ++t) fj = (t == j) ? f[t] : fj;
    if (__fsub_rn(fj, m) > __fmaf_rn(__fadd_rn(x2, __fadd_rn(m, fj)), 0x1p-16f, 0x1p-120f)) continue;
    const double e = score64(x, am, (uint32_t)b, s, tab);
    if (!have || e < be) {
      be = e;
      best = (uint32_t)b;
      have = true;
    }
  }
  if (want_err) *err = be;
  return best;
}

// floor(err * 2^P) as a 128-bit integer (err * 2^P < 2^87 by construction).
__device__ __forceinline__ void to_fixed(double err, double two_p, unsigned long long& lo, unsigned long long& hi) {
  const double w = __dmul_rn(err, two_p);
  const double h = floor(__dmul_rn(w, 0x1p-64));
  hi = __double2ull_rz(h);
  lo = __double2ull_rd(__fma_rn(h, -0x1p64, w));
}

__device__ __forceinline__ void add128(unsigned long long& lo, unsigned long long& hi, unsigned long long alo,
                                      unsigned long long ahi) {
  const unsigned long long l = lo + alo;
  hi += ahi + (l < alo ? 1ull : 0ull);
  lo = l;
}

// P = 80 - 2 floor(log2 amax) for a positive finite amax, as the fp64 2^P.
__device__ __forceinline__ double objective_scale(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const uint32_t f = (b >> 23) & 0xFFu;
  const int e = f != 0u ? (int)f - 127 : (31 - __clz((int)(b & 0x7FFFFFu))) - 149;
  const int P = 80 - 2 * e;
  return __longlong_as_double((long long)(P + 1023) << 52);
}

__global__ void __launch_bounds__(kThreads) mse_tensor_step_kernel(MseParams p) {
  __shared__ float2 tab[kTensorCands][128];
  __shared__ float sk[kTensorCands], yk[kTensorCands];
  __shared__ unsigned long long acc[kTensorCands][kWarps][2];
  __shared__ unsigned long long tot[kTensorCands][2];
  __shared__ bool last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_trigger();
  pdl_wait();
  const float s = start_scale(p);
  const float amax = *p.amax;
  const bool live = amax > 0.0f && amax <= 3.4028235e38f;
  for (int k = threadIdx.x; k < kTensorCands; k += blockDim.x) {
    sk[k] = step_scale(s, k);
    yk[k] = __frcp_rn(sk[k]);
  }
  __syncthreads();
  for (int k = 0; k < kTensorCands; ++k) nv_fill_scale_table(tab[k], sk[k]);
  for (int i = threadIdx.x; i < kTensorCands * kWarps * 2; i += blockDim.x) (&acc[0][0][0])[i] = 0ull;
  __syncthreads();
  if (live) {
    const double two_p = objective_scale(amax);
    // whole warps walk the blocks together (lanes past the end add zeros) so that each candidate's
    // 128-bit sum can be reduced across the warp
    for (uint32_t base = blockIdx.x * blockDim.x + 32u * warp; base < p.nblocks; base += gridDim.x * blockDim.x) {
      const uint32_t blk = base + lane;
      const bool ok = blk < p.nblocks;
      float x[16], am = 0.0f;
      if (ok) {
        load_block(p, blk, x, am);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.0f;
      }
#pragma unroll 1
      for (int k = 0; k < kTensorCands; ++k) {
        unsigned long long lo = 0ull, hi = 0ull;
        if (ok) {
          double err = 0.0;
          block_byte(x, am, sk[k], yk[k], recip_usable(sk[k]), tab[k], true, &err);
          to_fixed(err, two_p, lo, hi);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          add128(lo, hi, __shfl_down_sync(0xFFFFFFFFu, lo, off), __shfl_down_sync(0xFFFFFFFFu, hi, off));
        if (lane == 0) add128(acc[k][warp][0], acc[k][warp][1], lo, hi);
      }
    }
  }
  __syncthreads();
  // this CTA's sums, one thread per candidate, then the last CTA to finish picks the winner
  if (threadIdx.x < kTensorCands) {
    unsigned long long lo = 0ull, hi = 0ull;
    for (int w = 0; w < kWarps; ++w) add128(lo, hi, acc[threadIdx.x][w][0], acc[threadIdx.x][w][1]);
    p.partials[((size_t)blockIdx.x * kTensorCands + threadIdx.x) * 2] = lo;
    p.partials[((size_t)blockIdx.x * kTensorCands + threadIdx.x) * 2 + 1] = hi;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(p.ticket, 1u) == gridDim.x - 1u;
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (threadIdx.x < kTensorCands) {
    unsigned long long lo = 0ull, hi = 0ull;
    for (uint32_t c = 0; c < gridDim.x; ++c) {
      const unsigned long long* q = p.partials + ((size_t)c * kTensorCands + threadIdx.x) * 2;
      add128(lo, hi, __ldcg(q), __ldcg(q + 1));
    }
    tot[threadIdx.x][0] = lo;
    tot[threadIdx.x][1] = hi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // least Q; ties to the smallest |k|, then to k < 0 (k = index - 8)
    int best = kTensorCands / 2;
    for (int d = 1; d <= kTensorCands / 2; ++d) {
      for (int sg = -1; sg <= 1; sg += 2) {
        const int i = kTensorCands / 2 + sg * d;
        const bool less = tot[i][1] < tot[best][1] || (tot[i][1] == tot[best][1] && tot[i][0] < tot[best][0]);
        if (less) best = i;
      }
    }
    *p.s_t = live ? sk[best] : s;
    *p.ticket = 0u;                                    // ready for the next launch
  }
}

template <int RND, bool SFMMA>
__global__ void __launch_bounds__(kThreads) mse_quantize_kernel(MseParams p) {
  __shared__ float2 tab[128];
  pdl_trigger();
  pdl_wait();
  const float s = start_scale(p);
  nv_fill_scale_table(tab, s);
  __syncthreads();
  if (p.from_amax && blockIdx.x == 0 && threadIdx.x == 0) *p.s_t = s;
  const float y_s = __frcp_rn(s);
  const bool s_ok = recip_usable(s);
  for (uint32_t blk = blockIdx.x * blockDim.x + threadIdx.x; blk < p.nblocks; blk += gridDim.x * blockDim.x) {
    float x[16], am;
    load_block(p, blk, x, am);
    const uint32_t byte = block_byte(x, am, s, y_s, s_ok, tab, false, nullptr);
    uint32_t w[2] = {0u, 0u};
    if (byte != 0u) {
      nv_divide_block<RND, 16>(x, am, tab[byte], x);
      if (RND == 0) {
        w[0] = e2m1x4_rn(x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]);
        w[1] = e2m1x4_rn(x[8], x[9], x[10], x[11], x[12], x[13], x[14], x[15]);
      } else {
        const unsigned long long j0 = (unsigned long long)blk * 4u;        // Philox counter of element 16 blk
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const unsigned long long j = j0 + 2u * k;
          const u32x4 a = philox4x32_10((uint32_t)j, (uint32_t)(j >> 32), p.keys);
          const u32x4 b = philox4x32_10((uint32_t)(j + 1), (uint32_t)((j + 1) >> 32), p.keys);
          const float* xe = x + 8 * k;
          const uint32_t n[8] = {e2m1_sr(xe[0], a.x), e2m1_sr(xe[1], a.y), e2m1_sr(xe[2], a.z), e2m1_sr(xe[3], a.w),
                                 e2m1_sr(xe[4], b.x), e2m1_sr(xe[5], b.y), e2m1_sr(xe[6], b.z), e2m1_sr(xe[7], b.w)};
          w[k] = pack8_nibbles(n);
        }
      }
    }
    reinterpret_cast<uint2*>(p.codes)[blk] = make_uint2(w[0], w[1]);
    if (SFMMA) {
      const uint32_t row = blk / p.bpr;
      p.scales[sf_mma_offset(row, blk - row * p.bpr, p.g4)] = (uint8_t)byte;
    } else {
      p.scales[blk] = (uint8_t)byte;
    }
  }
}

template <typename K>
int resident(K kernel) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, 0) != cudaSuccess || n < 1) n = 1;
  return n;
}

}  // namespace

cudaError_t launch_quantize_mse(const QuantizeParams& q, float* ts_out, int iters, const Scratch& s, int num_sms,
                                cudaStream_t st) {
  MseParams p;
  p.x = static_cast<const uint16_t*>(q.x);
  p.ld = q.ld;
  p.nblocks = (uint32_t)(q.rows * (q.cols / 16));
  p.bpr = (uint32_t)(q.cols / 16);
  p.g4 = (uint32_t)((q.cols / 16 + 3) / 4);
  p.amax = s.mse_amax;
  p.s_t = ts_out;
  p.partials = s.mse_partials;
  p.ticket = s.mse_ticket;
  p.codes = q.codes;
  p.scales = q.scales;
  p.sf_mma = q.sf_mma;
  p.keys = philox_keys(q.seed);
  cudaError_t e = launch_amax(q.x, q.rows, q.cols, q.ld, 0, 0, s.mse_amax, s, num_sms, st);
  if (e != cudaSuccess) return e;
  const uint32_t want = (p.nblocks + kThreads - 1) / kThreads;
  static const int occ_t = resident(mse_tensor_step_kernel);
  uint32_t grid_t = (uint32_t)(num_sms * occ_t);
  if (grid_t > (uint32_t)kMaxMseCtas) grid_t = kMaxMseCtas;
  if (want < grid_t) grid_t = want > 0 ? want : 1;
  for (int it = 0; it < iters; ++it) {
    p.from_amax = it == 0;
    e = launch_kernel(mse_tensor_step_kernel, dim3(grid_t), dim3(kThreads), 0, st, false, 1u, p);
    if (e != cudaSuccess) return e;
  }
  p.from_amax = iters == 0;
  auto pick = [&](auto kernel) -> cudaError_t {
    static const int occ = resident(kernel);
    uint32_t grid = (uint32_t)(num_sms * occ);
    if (want < grid) grid = want > 0 ? want : 1;
    return launch_kernel(kernel, dim3(grid), dim3(kThreads), 0, st, false, 1u, p);
  };
  const bool sr = q.rnd == RND_SR;
  if (q.sf_mma) return sr ? pick(mse_quantize_kernel<1, true>) : pick(mse_quantize_kernel<0, true>);
  return sr ? pick(mse_quantize_kernel<1, false>) : pick(mse_quantize_kernel<0, false>);
}

}  // namespace fp4lib
