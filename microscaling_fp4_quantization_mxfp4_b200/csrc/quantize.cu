// Block-scaled FP4 quantization, block-Hadamard fused quantization, tensor
// amax and dequantization kernels for sm_100a.
//
// Method ("FP4 All the Way: Fully Quantized Training of LLMs", Abstract;
// "Bridging the Gap Between Promise and Performance for Microscaling FP4
// Quantization", Abstract and its summary post, item 3):
//   per block of 32 (MXFP4, power-of-two E8M0 scale) or 16 (NVFP4, E4M3 scale
//   under an fp32 tensor scale) elements along the contraction axis: block
//   absmax -> scale -> E2M1 codes by round-to-nearest-even or Philox
//   stochastic rounding, optionally after a block-diagonal Hadamard rotation.
//
// All of these are HBM-bound streaming kernels: 128-bit coalesced loads of
// bf16, warp-shuffle block maxima, packed 32-bit code stores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fp4_device.cuh"
#include "fp4_internal.h"

using namespace fp4dev;

namespace fp4lib {

FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  f.shift = s;
  f.mul = (uint32_t)((((1ull << s) - d) << 32) / d + 1ull);
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return (uint32_t)(((unsigned long long)__umulhi(n, f.mul) + n) >> f.shift);
}

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// ============================================================= amax pass ===
constexpr int kAmaxUnroll = 4;

struct AmaxParams {
  const uint16_t* x;
  uint32_t rows_x_cpr;   // number of 8-element chunks
  FastDiv cpr;           // chunks per row
  int64_t ld;
  int contig;            // ld == cols: chunk c starts at element 8c
  float* partials;
  unsigned* counter;
  float* out;
  int mode;
};

template <int HAD>
__global__ void __launch_bounds__(256) amax_kernel(AmaxParams p) {
  const int lane = threadIdx.x & 31;
  const uint32_t nchunks = p.rows_x_cpr;
  const uint32_t ntiles = (nchunks + 31u) >> 5;
  const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  float m = 0.0f;
  for (uint32_t t0 = gwarp; t0 < ntiles; t0 += nwarps * kAmaxUnroll) {
    uint4 v[kAmaxUnroll];
#pragma unroll
    for (int u = 0; u < kAmaxUnroll; ++u) {
      const uint32_t chunk = (t0 + (uint32_t)u * nwarps) * 32u + lane;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (t0 + (uint32_t)u * nwarps < ntiles && chunk < nchunks) {
        const uint32_t row = p.contig ? 0u : fdiv(chunk, p.cpr);
        const int64_t off = p.contig ? (int64_t)chunk * 8 : (int64_t)row * p.ld + (int64_t)(chunk - row * p.cpr.d) * 8;
        v[u] = ld_stream(p.x + off);
      }
    }
#pragma unroll
    for (int u = 0; u < kAmaxUnroll; ++u) {
      if (t0 + (uint32_t)u * nwarps >= ntiles) break;     // warp-uniform
      float x[8];
      unpack8(v[u], x);
      if (HAD) hadamard_rotate<HAD>(x, lane);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
    }
  }
  // non-negative floats order like their bit patterns
  uint32_t bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m));
  __shared__ uint32_t wmax[8];
  __shared__ bool is_last;
  if (lane == 0) wmax[threadIdx.x >> 5] = bits;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = max(b, wmax[w]);
    p.partials[blockIdx.x] = __uint_as_float(b);
    __threadfence();
    const unsigned ticket = atomicAdd(p.counter, 1u);
    is_last = (ticket == gridDim.x - 1);
  }
  __syncthreads();
  if (!is_last) return;
  // last CTA: combine the partial maxima (written by other CTAs, read past L1)
  uint32_t b = 0;
  for (uint32_t i = threadIdx.x; i < gridDim.x; i += blockDim.x)
    b = max(b, __float_as_uint(__ldcg(p.partials + i)));
  b = __reduce_max_sync(0xFFFFFFFFu, b);
  if (lane == 0) wmax[threadIdx.x >> 5] = b;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = max(r, wmax[w]);
    const float amax = __uint_as_float(r);
    if (p.mode == 0) {
      *p.out = amax;
    } else {
      *p.out = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
    }
    *p.counter = 0u;   // ready for the next call on this device
  }
}

__global__ void nv_tensor_scale_kernel(const float* amax, float* out) {
  const float a = *amax;
  *out = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);
}

// ======================================================== axis-1 quantize ===
struct QRowParams {
  const uint16_t* x;
  uint32_t nchunks;
  FastDiv cpr;           // chunks (8 elements) per row
  int64_t ld;
  int contig;            // ld == cols
  uint32_t cols;
  uint32_t g4;           // padded k-groups / 4 (tensor-core scale layout)
  unsigned long long seed;
  const float* ts;
  float* ts_copy_out;
  uint32_t* codes;       // [rows, cols/8] 32-bit words of 8 nibbles
  uint8_t* scales;
  float* rotated;
};

constexpr int kUnroll = 4;

template <int FMT, int RND, int HAD, bool SFMMA>
__device__ __forceinline__ void quantize_chunk(const QRowParams& p, const uint4 v, uint32_t chunk, bool valid,
                                               int lane, float s_t) {
  constexpr int LPB = FMT == FMT_MX ? 4 : 2;   // lanes per scale block
  float x[8];
  unpack8(v, x);
  if (HAD) {
    hadamard_rotate<HAD>(x, lane);
    if (p.rotated != nullptr && valid) {
      float4* r = reinterpret_cast<float4*>(p.rotated + (size_t)chunk * 8);
      r[0] = make_float4(x[0], x[1], x[2], x[3]);
      r[1] = make_float4(x[4], x[5], x[6], x[7]);
    }
  }
  float am = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(x[i]));
#pragma unroll
  for (int o = 1; o < LPB; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));

  uint32_t byte;
  bool zero;
  float v8[8];
  if (FMT == FMT_MX) {
    byte = mx_scale_byte(am);
    const float inv = mx_inv_scale(byte);
#pragma unroll
    for (int i = 0; i < 8; ++i) v8[i] = __fmul_rn(x[i], inv);     // exact power-of-two scaling
    zero = (am == 0.0f);
  } else {
    const float t = __fdiv_rn(__fdiv_rn(am, 6.0f), s_t);
    byte = e4m3_rn_sat(t);
    zero = (byte == 0u);
    const float S = zero ? 1.0f : __fmul_rn(e4m3_value(byte), s_t);
    const float y = __frcp_rn(S);
    bool ok = recip_usable(S);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      bool oki;
      v8[i] = div_by_recip(x[i], S, y, oki);
      ok = ok && oki;
    }
    if (__any_sync(0xFFFFFFFFu, !ok)) {       // rare: tiny values or scales -> IEEE division
      if (!ok) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v8[i] = __fdiv_rn(x[i], S);
      }
    }
  }
  uint32_t packed;
  if (RND == RND_RTN) {
    packed = pack8_rtn(v8);
  } else {
    uint32_t r[8];
    philox_words8((unsigned long long)chunk * 8ull, p.seed, r);
    packed = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) packed |= e2m1_sr(v8[i], r[i]) << (4 * i);
  }
  if (zero) packed = 0u;
  if (valid) {
    p.codes[chunk] = packed;
    if ((lane & (LPB - 1)) == 0) {
      if (SFMMA) {
        const uint32_t row = fdiv(chunk, p.cpr);
        const uint32_t g = (chunk - row * p.cpr.d) / LPB;
        p.scales[sf_mma_offset(row, g, p.g4)] = (uint8_t)byte;
      } else {
        p.scales[chunk / LPB] = (uint8_t)byte;
      }
    }
  }
}

template <int FMT, int RND, int HAD, bool SFMMA>
__global__ void __launch_bounds__(256) quantize_rows_kernel(QRowParams p) {
  const int lane = threadIdx.x & 31;
  const uint32_t ntiles = (p.nchunks + 31u) >> 5;
  const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  float s_t = 1.0f;
  if (FMT == FMT_NV) {
    s_t = *p.ts;
    if (p.ts_copy_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *p.ts_copy_out = s_t;
  }
  for (uint32_t t0 = gwarp; t0 < ntiles; t0 += nwarps * kUnroll) {
    uint4 v[kUnroll];
    uint32_t chunk[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t t = t0 + (uint32_t)u * nwarps;
      chunk[u] = t * 32u + lane;
      if (t < ntiles && chunk[u] < p.nchunks) {
        if (p.contig) {
          v[u] = ld_stream(p.x + (int64_t)chunk[u] * 8);
        } else {
          const uint32_t row = fdiv(chunk[u], p.cpr);
          const uint32_t c8 = chunk[u] - row * p.cpr.d;
          v[u] = ld_stream(p.x + (int64_t)row * p.ld + (int64_t)c8 * 8);
        }
      } else {
        v[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t t = t0 + (uint32_t)u * nwarps;
      if (t < ntiles)   // warp-uniform: every lane of the warp takes the same branch
        quantize_chunk<FMT, RND, HAD, SFMMA>(p, v[u], chunk[u], chunk[u] < p.nchunks, lane, s_t);
    }
  }
}

// ======================================================== axis-0 quantize ===
// Blocks run down the columns of x[R, C]; the output is written transposed
// (codes [C, R/2]).  A CTA stages a 128-row x 64-column bf16 tile in shared
// memory with coalesced 128-bit loads; each thread then owns one column and a
// 32-row segment (one MX block / two NV blocks) and writes its packed codes
// as one contiguous run of the output row.
struct QColParams {
  const uint16_t* x;
  uint32_t R, C;
  int64_t ld;
  uint32_t G, g4;        // k-groups per output row (R / block) and padded/4
  unsigned long long seed;
  const float* ts;
  float* ts_copy_out;
  uint8_t* codes;
  uint8_t* scales;
};

template <int FMT, int RND, bool SFMMA>
__global__ void __launch_bounds__(256) quantize_cols_kernel(QColParams p) {
  __shared__ __align__(16) uint16_t tile[128][64];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t tiles_r = (p.R + 127u) / 128u, tiles_c = (p.C + 63u) / 64u;
  float s_t = 1.0f;
  if (FMT == FMT_NV) {
    s_t = *p.ts;
    if (p.ts_copy_out != nullptr && blockIdx.x == 0 && tid == 0) *p.ts_copy_out = s_t;
  }
  for (uint32_t t = blockIdx.x; t < tiles_r * tiles_c; t += gridDim.x) {
    const uint32_t tc = t / tiles_r, tr = t - tc * tiles_r;
    const uint32_t r0 = tr * 128u, c0 = tc * 64u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + 256 * i, row = idx >> 3, ch = idx & 7;
      const uint32_t gr = r0 + row, gc = c0 + ch * 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (gr < p.R && gc < p.C) v = ld_stream(p.x + (int64_t)gr * p.ld + gc);
      *reinterpret_cast<uint4*>(&tile[row][ch * 8]) = v;
    }
    __syncthreads();
    const uint32_t c = c0 + 32u * (warp & 1) + lane;
    const uint32_t seg = warp >> 1;
    const uint32_t rbase = r0 + 32u * seg;
    if (c >= p.C || rbase >= p.R) continue;
    float xv[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) xv[i] = __uint_as_float((uint32_t)tile[32 * seg + i][32 * (warp & 1) + lane] << 16);
    constexpr int BS = FMT == FMT_MX ? 32 : 16;
    constexpr int NB = 32 / BS;
    uint32_t words[4];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const uint32_t rb = rbase + b * BS;
      if (rb >= p.R) break;
      float am = 0.0f;
#pragma unroll
      for (int i = 0; i < BS; ++i) am = fmaxf(am, fabsf(xv[b * BS + i]));
      uint32_t byte;
      bool zero;
      float inv = 1.0f, S = 1.0f, y = 1.0f;
      bool fast = true;
      if (FMT == FMT_MX) {
        byte = mx_scale_byte(am);
        inv = mx_inv_scale(byte);
        zero = (am == 0.0f);
      } else {
        const float tt = __fdiv_rn(__fdiv_rn(am, 6.0f), s_t);
        byte = e4m3_rn_sat(tt);
        zero = (byte == 0u);
        S = zero ? 1.0f : __fmul_rn(e4m3_value(byte), s_t);
        y = __frcp_rn(S);
        fast = recip_usable(S);
      }
#pragma unroll
      for (int w8 = 0; w8 < BS / 8; ++w8) {
        float v8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xi = xv[b * BS + w8 * 8 + i];
          if (FMT == FMT_MX) {
            v8[i] = __fmul_rn(xi, inv);
          } else {
            bool oki;
            v8[i] = div_by_recip(xi, S, y, oki);
            if (!(fast && oki)) v8[i] = __fdiv_rn(xi, S);
          }
        }
        uint32_t packed;
        if (RND == RND_RTN) {
          packed = pack8_rtn(v8);
        } else {
          packed = 0u;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const unsigned long long idx = (unsigned long long)(rb + w8 * 8 + i) * p.C + c;
            packed |= e2m1_sr(v8[i], philox_word(idx, p.seed)) << (4 * i);
          }
        }
        words[b * (BS / 8) + w8] = zero ? 0u : packed;
      }
      const uint32_t g = rb / BS;
      if (SFMMA) p.scales[sf_mma_offset(c, g, p.g4)] = (uint8_t)byte;
      else p.scales[(size_t)c * p.G + g] = (uint8_t)byte;
      if (FMT == FMT_NV) {
        *reinterpret_cast<uint2*>(p.codes + (size_t)c * (p.R / 2) + rb / 2) = make_uint2(words[2 * b], words[2 * b + 1]);
      }
    }
    if (FMT == FMT_MX) {
      *reinterpret_cast<uint4*>(p.codes + (size_t)c * (p.R / 2) + rbase / 2) =
          make_uint4(words[0], words[1], words[2], words[3]);
    }
  }
}

// ============================================================ dequantize ===
struct DeqParams {
  const uint32_t* codes;  // 32-bit words of 8 nibbles
  const uint8_t* scales;
  const float* ts;
  uint32_t nchunks;
  FastDiv cpr;
  uint32_t g4;
  void* out;
};

template <int FMT, bool SFMMA, bool BF16>
__device__ __forceinline__ void dequantize_chunk(const DeqParams& p, uint32_t chunk, uint32_t w, float s_t) {
  constexpr int LPB = FMT == FMT_MX ? 4 : 2;
  uint32_t byte;
  if (SFMMA) {
    const uint32_t row = fdiv(chunk, p.cpr);
    byte = p.scales[sf_mma_offset(row, (chunk - row * p.cpr.d) / LPB, p.g4)];
  } else {
    byte = p.scales[chunk / LPB];
  }
  float y[8];
  if (FMT == FMT_MX) {
    const float sc = mx_scale_value(byte);
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(e2m1_value((w >> (4 * i)) & 0xFu), sc);
  } else {
    const float sb = e4m3_value(byte);
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fmul_rn(__fmul_rn(e2m1_value((w >> (4 * i)) & 0xFu), sb), s_t);
  }
  if (BF16) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(y[2 * i]));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(y[2 * i + 1]));
      o[i] = lo | (hi << 16);
    }
    reinterpret_cast<uint4*>(p.out)[chunk] = make_uint4(o[0], o[1], o[2], o[3]);
  } else {
    float4* o = reinterpret_cast<float4*>(p.out) + (size_t)chunk * 2;
    o[0] = make_float4(y[0], y[1], y[2], y[3]);
    o[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
}

// Each thread takes two adjacent chunks (16 codes, one 8-byte load) per step;
// the chunk count is even because rows hold a whole number of 16-element blocks.
template <int FMT, bool SFMMA, bool BF16>
__global__ void __launch_bounds__(256) dequantize_kernel(DeqParams p) {
  const float s_t = FMT == FMT_NV ? *p.ts : 1.0f;
  const uint32_t npairs = p.nchunks / 2;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < npairs; i += 2 * stride) {
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(p.codes) + i);
    const bool has2 = i + stride < npairs;
    uint2 b = make_uint2(0u, 0u);
    if (has2) b = __ldg(reinterpret_cast<const uint2*>(p.codes) + i + stride);
    dequantize_chunk<FMT, SFMMA, BF16>(p, 2 * i, a.x, s_t);
    dequantize_chunk<FMT, SFMMA, BF16>(p, 2 * i + 1, a.y, s_t);
    if (has2) {
      dequantize_chunk<FMT, SFMMA, BF16>(p, 2 * (i + stride), b.x, s_t);
      dequantize_chunk<FMT, SFMMA, BF16>(p, 2 * (i + stride) + 1, b.y, s_t);
    }
  }
}

// ============================================================== launchers ===
template <typename K>
static int resident_ctas(K kernel, int threads) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1) n = 1;
  return n;
}

template <int HAD>
static cudaError_t amax_launch(const AmaxParams& ap, uint32_t ntiles, int num_sms, cudaStream_t st) {
  static int occ = resident_ctas(amax_kernel<HAD>, 256);
  uint32_t want = (ntiles + 8u * kAmaxUnroll - 1u) / (8u * kAmaxUnroll);
  uint32_t grid = (uint32_t)num_sms * (uint32_t)occ;
  if (grid > (uint32_t)kMaxAmaxBlocks) grid = kMaxAmaxBlocks;
  if (want < grid) grid = want > 0 ? want : 1;
  amax_kernel<HAD><<<grid, 256, 0, st>>>(ap);
  return cudaGetLastError();
}

cudaError_t launch_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, int had, int mode, float* out,
                        const Scratch& s, int num_sms, cudaStream_t st) {
  AmaxParams ap;
  ap.x = static_cast<const uint16_t*>(x);
  ap.rows_x_cpr = (uint32_t)(rows * (cols / 8));
  ap.cpr = make_fastdiv((uint32_t)(cols / 8));
  ap.ld = ld;
  ap.contig = (ld == cols);
  ap.partials = s.partials;
  ap.counter = s.counter;
  ap.out = out;
  ap.mode = mode;
  const uint32_t ntiles = (ap.rows_x_cpr + 31u) / 32u;
  switch (had) {
    case 0: return amax_launch<0>(ap, ntiles, num_sms, st);
    case 16: return amax_launch<16>(ap, ntiles, num_sms, st);
    case 32: return amax_launch<32>(ap, ntiles, num_sms, st);
    case 64: return amax_launch<64>(ap, ntiles, num_sms, st);
    case 128: return amax_launch<128>(ap, ntiles, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_amax_fixed_grid(const void* x, int64_t rows, int64_t cols, int64_t ld, float* out,
                                   const Scratch& s, uint32_t grid, cudaStream_t st) {
  AmaxParams ap;
  ap.x = static_cast<const uint16_t*>(x);
  ap.rows_x_cpr = (uint32_t)(rows * (cols / 8));
  ap.cpr = make_fastdiv((uint32_t)(cols / 8));
  ap.ld = ld;
  ap.contig = (ld == cols);
  ap.partials = s.partials;
  ap.counter = s.counter;
  ap.out = out;
  ap.mode = 0;
  amax_kernel<0><<<grid, 256, 0, st>>>(ap);
  return cudaGetLastError();
}

cudaError_t launch_nv_tensor_scale(const float* amax, float* out, cudaStream_t st) {
  nv_tensor_scale_kernel<<<1, 1, 0, st>>>(amax, out);
  return cudaGetLastError();
}

template <int FMT, int RND, int HAD, bool SFMMA>
static cudaError_t rows_launch(const QRowParams& qp, int num_sms, cudaStream_t st) {
  static int occ = resident_ctas(quantize_rows_kernel<FMT, RND, HAD, SFMMA>, 256);
  const uint32_t ntiles = (qp.nchunks + 31u) / 32u;
  uint32_t want = (ntiles + 8u * kUnroll - 1u) / (8u * kUnroll);
  uint32_t grid = (uint32_t)num_sms * (uint32_t)occ;
  if (want < grid) grid = want > 0 ? want : 1;
  quantize_rows_kernel<FMT, RND, HAD, SFMMA><<<grid, 256, 0, st>>>(qp);
  return cudaGetLastError();
}

template <int FMT, int RND, int HAD>
static cudaError_t rows_dispatch_sf(const QRowParams& qp, bool sfmma, int num_sms, cudaStream_t st) {
  return sfmma ? rows_launch<FMT, RND, HAD, true>(qp, num_sms, st) : rows_launch<FMT, RND, HAD, false>(qp, num_sms, st);
}

template <int FMT, int RND>
static cudaError_t rows_dispatch_had(const QRowParams& qp, int had, bool sfmma, int num_sms, cudaStream_t st) {
  switch (had) {
    case 0: return rows_dispatch_sf<FMT, RND, 0>(qp, sfmma, num_sms, st);
    case 16: return rows_dispatch_sf<FMT, RND, 16>(qp, sfmma, num_sms, st);
    case 32: return rows_dispatch_sf<FMT, RND, 32>(qp, sfmma, num_sms, st);
    case 64: return rows_dispatch_sf<FMT, RND, 64>(qp, sfmma, num_sms, st);
    case 128: return rows_dispatch_sf<FMT, RND, 128>(qp, sfmma, num_sms, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int FMT, int RND, bool SFMMA>
static cudaError_t cols_launch(const QColParams& qp, int num_sms, cudaStream_t st) {
  static int occ = resident_ctas(quantize_cols_kernel<FMT, RND, SFMMA>, 256);
  const uint32_t ntiles = ((qp.R + 127u) / 128u) * ((qp.C + 63u) / 64u);
  uint32_t grid = (uint32_t)num_sms * (uint32_t)occ;
  if (ntiles < grid) grid = ntiles > 0 ? ntiles : 1;
  quantize_cols_kernel<FMT, RND, SFMMA><<<grid, 256, 0, st>>>(qp);
  return cudaGetLastError();
}

template <int FMT, int RND>
static cudaError_t cols_dispatch(const QColParams& qp, bool sfmma, int num_sms, cudaStream_t st) {
  return sfmma ? cols_launch<FMT, RND, true>(qp, num_sms, st) : cols_launch<FMT, RND, false>(qp, num_sms, st);
}

cudaError_t launch_quantize(const QuantizeParams& p, int num_sms, cudaStream_t st) {
  const int bs = p.fmt == FMT_MX ? 32 : 16;
  const bool sfmma = p.sf_mma != 0;
  if (p.axis == 1) {
    QRowParams qp;
    qp.x = static_cast<const uint16_t*>(p.x);
    qp.nchunks = (uint32_t)(p.rows * (p.cols / 8));
    qp.cpr = make_fastdiv((uint32_t)(p.cols / 8));
    qp.ld = p.ld;
    qp.contig = (p.ld == p.cols);
    qp.cols = (uint32_t)p.cols;
    qp.g4 = (uint32_t)((p.cols / bs + 3) / 4);
    qp.seed = p.seed;
    qp.ts = p.ts;
    qp.ts_copy_out = p.ts_copy_out;
    qp.codes = reinterpret_cast<uint32_t*>(p.codes);
    qp.scales = p.scales;
    qp.rotated = p.rotated;
    if (p.fmt == FMT_MX)
      return p.rnd == RND_RTN ? rows_dispatch_had<FMT_MX, RND_RTN>(qp, p.had, sfmma, num_sms, st)
                              : rows_dispatch_had<FMT_MX, RND_SR>(qp, p.had, sfmma, num_sms, st);
    return p.rnd == RND_RTN ? rows_dispatch_had<FMT_NV, RND_RTN>(qp, p.had, sfmma, num_sms, st)
                            : rows_dispatch_had<FMT_NV, RND_SR>(qp, p.had, sfmma, num_sms, st);
  }
  QColParams qp;
  qp.x = static_cast<const uint16_t*>(p.x);
  qp.R = (uint32_t)p.rows;
  qp.C = (uint32_t)p.cols;
  qp.ld = p.ld;
  qp.G = (uint32_t)(p.rows / bs);
  qp.g4 = (qp.G + 3u) / 4u;
  qp.seed = p.seed;
  qp.ts = p.ts;
  qp.ts_copy_out = p.ts_copy_out;
  qp.codes = p.codes;
  qp.scales = p.scales;
  if (p.fmt == FMT_MX)
    return p.rnd == RND_RTN ? cols_dispatch<FMT_MX, RND_RTN>(qp, sfmma, num_sms, st)
                            : cols_dispatch<FMT_MX, RND_SR>(qp, sfmma, num_sms, st);
  return p.rnd == RND_RTN ? cols_dispatch<FMT_NV, RND_RTN>(qp, sfmma, num_sms, st)
                          : cols_dispatch<FMT_NV, RND_SR>(qp, sfmma, num_sms, st);
}

template <int FMT, bool SFMMA, bool BF16>
static cudaError_t deq_launch(const DeqParams& dp, int num_sms, cudaStream_t st) {
  static int occ = resident_ctas(dequantize_kernel<FMT, SFMMA, BF16>, 256);
  uint32_t want = (dp.nchunks / 2 + 511u) / 512u;
  uint32_t grid = (uint32_t)num_sms * (uint32_t)occ;
  if (want < grid) grid = want > 0 ? want : 1;
  dequantize_kernel<FMT, SFMMA, BF16><<<grid, 256, 0, st>>>(dp);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* ts, int64_t rows,
                              int64_t cols, int fmt, int sf_mma, void* out, int out_bf16, int num_sms,
                              cudaStream_t st) {
  const int bs = fmt == FMT_MX ? 32 : 16;
  DeqParams dp;
  dp.codes = reinterpret_cast<const uint32_t*>(codes);
  dp.scales = scales;
  dp.ts = ts;
  dp.nchunks = (uint32_t)(rows * (cols / 8));
  dp.cpr = make_fastdiv((uint32_t)(cols / 8));
  dp.g4 = (uint32_t)((cols / bs + 3) / 4);
  dp.out = out;
  const int key = (fmt == FMT_NV ? 4 : 0) | (sf_mma ? 2 : 0) | (out_bf16 ? 1 : 0);
  switch (key) {
    case 0: return deq_launch<FMT_MX, false, false>(dp, num_sms, st);
    case 1: return deq_launch<FMT_MX, false, true>(dp, num_sms, st);
    case 2: return deq_launch<FMT_MX, true, false>(dp, num_sms, st);
    case 3: return deq_launch<FMT_MX, true, true>(dp, num_sms, st);
    case 4: return deq_launch<FMT_NV, false, false>(dp, num_sms, st);
    case 5: return deq_launch<FMT_NV, false, true>(dp, num_sms, st);
    case 6: return deq_launch<FMT_NV, true, false>(dp, num_sms, st);
    default: return deq_launch<FMT_NV, true, true>(dp, num_sms, st);
  }
}

}  // namespace fp4lib
