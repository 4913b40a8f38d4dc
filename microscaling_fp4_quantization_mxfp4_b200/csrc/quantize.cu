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
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

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
  pdl_trigger();
  pdl_wait();
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
  pdl_trigger();
  pdl_wait();
  const float a = *amax;
  *out = (a == 0.0f) ? 1.0f : __fdiv_rn(a, 2688.0f);
}

// ======================================================== axis-1 quantize ===
struct QRowParams {
  const uint16_t* x;
  uint32_t nchunks;
  uint32_t nblocks;      // scale blocks (rows * cols / block)
  FastDiv bpr;           // scale blocks per row
  FastDiv cpr;           // chunks (8 elements) per row
  int64_t ld;
  int contig;            // ld == cols
  uint32_t cols;
  uint32_t g4;           // padded k-groups / 4 (tensor-core scale layout)
  unsigned long long seed;
  PhiloxKeys keys;      // the seed's Philox key schedule
  uint32_t mx_thr;      // MXFP4 exponent clip threshold (significand field; kMxClipOcp: the OCP rule)
  const float* ts;
  float* ts_copy_out;
  uint32_t* codes;       // [rows, cols/8] 32-bit words of 8 nibbles
  uint8_t* scales;
  float* rotated;
  unsigned* error;       // device error word (streaming kernels: bit 2 = a ring wait expired)
  void* deq;             // DQ kernels: the dequantized values [rows, cols] (fp32, or bf16 for DQ = 2)
  uint32_t sf_rows;      // tensor-core scale layout: valid rows and scale groups per row, whose padding
  uint32_t sf_groups;    // bytes (rows up to 128, groups up to 4 g4) the kernel writes as 0
  FastDiv g4d;           // division by g4
  unsigned long long jbase;  // Philox counter of the first element (row shards: first_row * cols / 4)
};

// Zero the tensor-core scale layout's padding (rows sf_rows .. multiple of 128, groups sf_groups ..
// 4 g4), dealt over the grid's threads `t` of `nt`; the valid bytes are the quantizer's.  A padding
// row's four groups 4j .. 4j + 3 are one aligned 32-bit word (one store each when the buffer is
// 4-byte aligned); the groups past sf_groups of valid rows (fewer than 4) are single bytes.  32-bit
// indices with the precomputed division by g4 (a 64-bit division per byte made the padding of a
// one-row activation cost about 10 us on a single CTA).
__device__ __forceinline__ void sf_pad_zero(const QRowParams& p, uint32_t t, uint32_t nt) {
  const uint32_t g4 = p.g4, gp = 4u * g4;
  const uint32_t rpad = ((p.sf_rows + 127u) & ~127u) - p.sf_rows;  // padding rows
  const uint32_t gpad = gp - p.sf_groups;                          // padding groups of valid rows
  if ((reinterpret_cast<uintptr_t>(p.scales) & 3u) == 0u) {
    for (uint32_t i = t; i < rpad * g4; i += nt) {
      const uint32_t k = fdiv(i, p.g4d), r = p.sf_rows + k, j = i - k * g4;
      *reinterpret_cast<uint32_t*>(p.scales + sf_mma_offset(r, 4u * j, g4)) = 0u;
    }
  } else {
    for (uint32_t i = t; i < rpad * gp; i += nt) {
      const uint32_t k = i / gp;
      p.scales[sf_mma_offset(p.sf_rows + k, i - k * gp, g4)] = 0u;
    }
  }
  for (uint32_t i = t; i < p.sf_rows * gpad; i += nt) {
    const uint32_t r = i / gpad;
    p.scales[sf_mma_offset(r, p.sf_groups + (i - r * gpad), g4)] = 0u;
  }
}

// Per-thread NVFP4 constants: the tensor scale, its reciprocal and the (S, 1/S) table.
struct NvConsts {
  float s_t;
  double yd_st;          // RN64(1 / s_t)
  const double* tabd;    // per E4M3 byte: RN64(1 / S), or (S, RN32(1 / S)) as a float2 (PAIRS)
};

// The per-CTA NVFP4 constants under tensor scale s_t: fills the 1 KB divisor table (every thread
// of the CTA takes part; visible after the caller's next __syncthreads).  PAIRS: the table holds
// (S, RN32(1 / S)) pairs for nv_divide_block2, else the fp64 reciprocals of div_by_recip64.
template <bool PAIRS = false>
__device__ __forceinline__ NvConsts nv_consts(float s_t, double* tabd) {
  if (PAIRS) {
    nv_fill_scale_table(reinterpret_cast<float2*>(tabd), s_t);
  } else {
    nv_fill_recip64_table(tabd, s_t);
  }
  return NvConsts{s_t, __drcp_rn((double)s_t), tabd};
}

// Whether quantize_block divides NVFP4 blocks with the pair table (nv_divide_block2), by measured
// speed: round-to-nearest (single-pass 4096^2 quantize + dequantize 28.8 -> 27.7 us) and stochastic
// rounding with the fused dequantize (36.6 -> 35.7 us).  Stochastic rounding alone, whose
// per-element range test then costs more than the conversions it saves, keeps the fp64
// reciprocals, as do four-over-six, axis-0 and 2-D blocks.
template <int FMT, int RND, int DQ>
constexpr bool kNvPairs = FMT == FMT_NV && (RND == RND_RTN || DQ != 0);

// One thread quantizes one whole scale block of E = 32 (MX) or 16 (NV)
// elements held as E/8 uint4: the block maximum, the scale and every division
// are computed once per block, with E independent element computations.
// (Splitting an MXFP4 block over a lane pair, 16 elements a thread at 31 warps,
// measured slower: 52.8 vs 48.5 us for SR and 17.8 vs 16.3 us for RTN at
// 8192 x 4096, since the per-block work is then done twice.)
template <int FMT>
struct BlockShape {
  static constexpr int E = FMT == FMT_MX ? 32 : 16;   // elements per block
  static constexpr int V = E / 8;                      // uint4 per block
};

// Four-over-six ("Four Over Six", Abstract): of the standard scale byte byte6 (block max -> 6) and
// the max -> 4 byte, the block takes the one whose round-to-nearest result has the lower squared
// error, sum over the block of (x - dequantized)^2 in fp64 added in element order; ties keep
// byte6, and a zero or identical max -> 4 byte is never taken.  x is replaced by its quotients
// under the chosen scale (exact where the rounding mode needs them) and the byte is returned.
//
// The two sums are first screened in fp32 (one fma per element and candidate).  Each fp32 sum is
// within 18 u (u = 2^-24) of the exact one, relatively, plus 16 * 2^-150 from underflow; each
// fp64 sum within 15 * 2^-53 (its terms are exact: x has 8 significant bits, the dequantized d at
// most 24, a non-zero d lies within a factor of 2 of x, so x - d has at most 26 bits and its
// square at most 52).  A screen gap above 2^-17 of the sums plus 2^-120 therefore decides the
// fp64 comparison; anything closer (near-ties, non-finite or tiny sums) takes the fp64 sums.
template <int RND, int E>
__device__ __forceinline__ uint32_t nv_four_over_six(float (&x)[E], float am, uint32_t byte6, const NvConsts& nv) {
  const float s_t = nv.s_t;
  float q6[E];
  nv_divide_block64<E>(x, nv.tabd[byte6], q6);
  const uint32_t byte4 = e4m3_rn_sat(nv_scale_arg4_64(am, s_t, nv.yd_st));
  bool pick4 = false;
  if (byte4 != byte6 && byte4 != 0u) {
    float q4[E];
    nv_divide_block64<E>(x, nv.tabd[byte4], q4);
    const __half2 g6 = __float2half2_rn(e4m3_value(byte6)), g4 = __float2half2_rn(e4m3_value(byte4));
    float f6 = 0.0f, f4 = 0.0f;
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      const float2 d6 = nv_rtn_dequant2(q6[i], q6[i + 1], g6, s_t);
      const float2 d4 = nv_rtn_dequant2(q4[i], q4[i + 1], g4, s_t);
      float e = __fsub_rn(x[i], d6.x);
      f6 = __fmaf_rn(e, e, f6);
      e = __fsub_rn(x[i], d4.x);
      f4 = __fmaf_rn(e, e, f4);
      e = __fsub_rn(x[i + 1], d6.y);
      f6 = __fmaf_rn(e, e, f6);
      e = __fsub_rn(x[i + 1], d4.y);
      f4 = __fmaf_rn(e, e, f4);
    }
    const float tol = __fmaf_rn(__fadd_rn(f4, f6), 0x1p-17f, 0x1p-120f);
    if (__fadd_rn(f4, tol) < f6) {
      pick4 = true;
    } else if (!(__fadd_rn(f6, tol) < f4)) {     // too close to call in fp32: the fp64 sums
      double acc6 = 0.0, acc4 = 0.0;
#pragma unroll
      for (int i = 0; i < E; i += 2) {
        const float2 d6 = nv_rtn_dequant2(q6[i], q6[i + 1], g6, s_t);
        const float2 d4 = nv_rtn_dequant2(q4[i], q4[i + 1], g4, s_t);
        const double x0 = (double)x[i], x1 = (double)x[i + 1];
        double e = __dsub_rn(x0, (double)d6.x);
        acc6 = __fma_rn(e, e, acc6);
        e = __dsub_rn(x0, (double)d4.x);
        acc4 = __fma_rn(e, e, acc4);
        e = __dsub_rn(x1, (double)d6.y);
        acc6 = __fma_rn(e, e, acc6);
        e = __dsub_rn(x1, (double)d4.y);
        acc4 = __fma_rn(e, e, acc4);
      }
      pick4 = acc4 < acc6;
    }
    if (pick4) {
#pragma unroll
      for (int i = 0; i < E; ++i) x[i] = q4[i];
    }
  }
  if (!pick4) {
#pragma unroll
    for (int i = 0; i < E; ++i) x[i] = q6[i];
  }
  return pick4 ? byte4 : byte6;
}

// Dequantized values of one block's packed codes w (E/8 words) under scale byte `byte`, as
// fp4_dequantize computes them (NVFP4: fp32(fp32(G[c] * sb) * s_t) with the exact f16 product;
// MXFP4: G[c] * 2^E), stored at element blk * E of the row-major output: fp32 (DQ = 1) or bf16
// (DQ = 2, round to nearest even).
template <int FMT, int DQ>
__device__ __forceinline__ void dequant_block_out(const QRowParams& p, const uint32_t* w, uint32_t byte, uint32_t blk,
                                                  float s_t) {
  constexpr int E = BlockShape<FMT>::E;
  float y[E];
  const __half2 sb = __float2half2_rn(FMT == FMT_MX ? 1.0f : e4m3_value(byte));
  const float sc = FMT == FMT_MX ? mx_scale_value(byte) : s_t;
#pragma unroll
  for (int k = 0; k < E / 8; ++k) {
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w[k]));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 hv = *reinterpret_cast<const __half2*>(&h[i]);
      const float2 g = __half22float2(FMT == FMT_MX ? hv : __hmul2(hv, sb));
      const float2 r = mul2(g, splat2(sc));
      y[8 * k + 2 * i] = r.x;
      y[8 * k + 2 * i + 1] = r.y;
    }
  }
  // 32-byte stores (one whole L2 sector per lane) when the output base allows them: a block's
  // values start at a multiple of 32 bytes.  16-byte stores from neighbouring lanes 64 bytes
  // apart would each half-fill a sector.
  const bool wide = (reinterpret_cast<uintptr_t>(p.deq) & 31u) == 0;
  uint32_t o32[DQ == 1 ? E : E / 2];
  if (DQ == 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) o32[i] = __float_as_uint(y[i]);
  } else {
#pragma unroll
    for (int i = 0; i < E / 2; ++i)
      o32[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y[2 * i])) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y[2 * i + 1])) << 16);
  }
  constexpr int W = DQ == 1 ? E : E / 2;                   // 32-bit words of the block's output
  uint32_t* o = static_cast<uint32_t*>(p.deq) + (size_t)blk * W;
  if (wide) {
#pragma unroll
    for (int k = 0; k < W / 8; ++k)
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(o + 8 * k), "r"(o32[8 * k]),
                   "r"(o32[8 * k + 1]), "r"(o32[8 * k + 2]), "r"(o32[8 * k + 3]), "r"(o32[8 * k + 4]),
                   "r"(o32[8 * k + 5]), "r"(o32[8 * k + 6]), "r"(o32[8 * k + 7])
                   : "memory");
  } else {
#pragma unroll
    for (int k = 0; k < W / 4; ++k)
      reinterpret_cast<uint4*>(o)[k] = make_uint4(o32[4 * k], o32[4 * k + 1], o32[4 * k + 2], o32[4 * k + 3]);
  }
}

// The lane bits that select a block's chunk order (chunk_swap): bit 2 for NVFP4, bits 1-2 for MXFP4.
template <int FMT> constexpr int kSwShift = FMT == FMT_MX ? 1 : 2;
template <int FMT> constexpr uint32_t kSwMask = FMT == FMT_MX ? 3u : FMT == FMT_NV ? 1u : 0u;

// Chunk order of a block as the shared-memory streaming kernels load it: register k holds the
// block's 16-byte chunk k ^ sw, with sw = bit 2 of the lane for NVFP4 (two chunks) and bits 1-2 for
// MXFP4 (four chunks), so that the eight lanes of a quarter warp read eight distinct 16-byte bank
// groups (in chunk order the 32- or 64-byte blocks of those lanes share banks: 2- or 4-way
// conflicts).  quantize_block puts the codes (and dequantized values) back in chunk order before
// they leave, and the rotation's butterflies follow the order (hadamard_rotate_block).  0 for
// four-over-six, which adds its error terms in element order.
template <int FMT, int HAD>
__device__ __forceinline__ uint32_t chunk_swap(int lane) {
  return FMT == FMT_NV ? (uint32_t)(lane >> kSwShift<FMT>) & kSwMask<FMT>
                       : FMT == FMT_MX ? (uint32_t)(lane >> kSwShift<FMT>) & kSwMask<FMT> : 0u;
}

// v[k] holds the block's chunk k ^ sw: SWZ = true with sw = chunk_swap(lane) in the streaming
// kernels (every lane's order set by its lane bits), SWZ = false and sw = 0 elsewhere.
template <int FMT, int RND, int HAD, bool SFMMA, int DQ = 0, bool SWZ = false>
__device__ __forceinline__ void quantize_block(const QRowParams& p, const uint4 (&v)[BlockShape<FMT>::V], uint32_t blk,
                                               bool valid, int lane, const NvConsts& nv, uint32_t sw = 0u) {
  constexpr int E = BlockShape<FMT>::E, V = BlockShape<FMT>::V;
  float x[E];
#pragma unroll
  for (int k = 0; k < V; ++k) {
    float t8[8];
    unpack8(v[k], t8);
#pragma unroll
    for (int i = 0; i < 8; ++i) x[8 * k + i] = t8[i];
  }
  if (HAD) {
    hadamard_rotate_block<HAD, E, kSwShift<FMT>, (SWZ ? (int)kSwMask<FMT> : 0)>(x, lane, sw);
    if (p.rotated != nullptr && valid) {
      float4* r = reinterpret_cast<float4*>(p.rotated + (size_t)blk * E);
#pragma unroll
      for (int k = 0; k < E / 4; ++k) {
        const uint32_t q = (((uint32_t)(k >> 1) ^ sw) << 1) | (uint32_t)(k & 1);   // chunk k/2 is chunk k/2 ^ sw
        r[q] = make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]);
      }
    }
  }
  float am = 0.0f;
#pragma unroll
  for (int i = 0; i < E; ++i) am = fmaxf(am, fabsf(x[i]));
  uint32_t byte;
  bool zero;
  if (FMT == FMT_MX) {
    byte = mx_scale_byte_clip(am, p.mx_thr);
    const float2 inv = splat2(mx_inv_scale(byte));
#pragma unroll
    for (int i = 0; i < E / 2; ++i) {                                   // exact power-of-two scaling
      const float2 t = mul2(make_float2(x[i], x[i + E / 2]), inv);
      x[i] = t.x;
      x[i + E / 2] = t.y;
    }
    zero = (am == 0.0f);
  } else {
    byte = e4m3_rn_sat(nv_scale_arg64(am, nv.s_t, nv.yd_st));
    if (FMT == FMT_NV46) {
      byte = nv_four_over_six<RND, E>(x, am, byte, nv);
    } else {
      if (kNvPairs<FMT, RND, DQ>) {
        nv_divide_block2<RND, E>(x, am, reinterpret_cast<const float2*>(nv.tabd)[byte]);
      } else {
        nv_divide_block64<E>(x, nv.tabd[byte], x);
      }
    }
    zero = (byte == 0u);
  }
  uint32_t w[E / 8];
  if (RND == RND_RTN) {
#pragma unroll
    for (int k = 0; k < E / 8; ++k)
      w[k] = e2m1x4_rn(x[8 * k], x[8 * k + 1], x[8 * k + 2], x[8 * k + 3], x[8 * k + 4], x[8 * k + 5], x[8 * k + 6],
                       x[8 * k + 7]);
  } else {
    const unsigned long long j0 = p.jbase + (unsigned long long)blk * (E / 4);   // counter of element blk*E
#pragma unroll
    for (int k = 0; k < E / 8; ++k) {
      const unsigned long long j = j0 + 2u * ((uint32_t)k ^ sw);          // slot k holds chunk k ^ sw
      const u32x4 a = philox4x32_10((uint32_t)j, (uint32_t)(j >> 32), p.keys);
      const u32x4 b = philox4x32_10((uint32_t)(j + 1), (uint32_t)((j + 1) >> 32), p.keys);
      const float* xe = x + 8 * k;
      const uint32_t n[8] = {e2m1_sr(xe[0], a.x), e2m1_sr(xe[1], a.y), e2m1_sr(xe[2], a.z), e2m1_sr(xe[3], a.w),
                             e2m1_sr(xe[4], b.x), e2m1_sr(xe[5], b.y), e2m1_sr(xe[6], b.z), e2m1_sr(xe[7], b.w)};
      w[k] = pack8_nibbles(n);
    }
  }
  if (FMT != FMT_NV46) {                                  // back to chunk order: w[c] <- w[c ^ sw]
    if (sw & 1u) {
#pragma unroll
      for (int k = 0; k < E / 8; k += 2) {
        const uint32_t t = w[k];
        w[k] = w[k + 1];
        w[k + 1] = t;
      }
    }
    if (E / 8 == 4 && (sw & 2u)) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint32_t t = w[k];
        w[k] = w[k + 2 < E / 8 ? k + 2 : k];
        w[k + 2 < E / 8 ? k + 2 : k] = t;
      }
    }
  }
  if (!valid) return;
  if (zero) {
#pragma unroll
    for (int k = 0; k < E / 8; ++k) w[k] = 0u;
  }
  if (FMT == FMT_MX) {
    reinterpret_cast<uint4*>(p.codes)[blk] = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    reinterpret_cast<uint2*>(p.codes)[blk] = make_uint2(w[0], w[1]);
  }
  if (DQ != 0) dequant_block_out<FMT, DQ>(p, w, byte, blk, nv.s_t);
  if (SFMMA) {
    const uint32_t row = fdiv(blk, p.bpr);
    p.scales[sf_mma_offset(row, blk - row * p.bpr.d, p.g4)] = (uint8_t)byte;
  } else {
    p.scales[blk] = (uint8_t)byte;
  }
}

// Strided inputs (ld != cols): one thread per scale block, loads straight from global memory.
template <int FMT, int RND, int HAD, bool SFMMA, int DQ = 0>
__global__ void __launch_bounds__(256) quantize_rows_kernel(QRowParams p) {
  pdl_trigger();
  constexpr int V = BlockShape<FMT>::V;
  __shared__ double tabd[128];
  const int lane = threadIdx.x & 31;
  pdl_wait();
  if (SFMMA) sf_pad_zero(p, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
  NvConsts nv{1.0f, 1.0, tabd};
  if (FMT != FMT_MX) {
    nv = nv_consts<kNvPairs<FMT, RND, DQ>>(*p.ts, tabd);
    if (p.ts_copy_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *p.ts_copy_out = nv.s_t;
    __syncthreads();
  }
  const uint32_t nunits = (p.nblocks + 31u) >> 5;               // warp units of 32 blocks
  const uint32_t gwarp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t u = gwarp; u < nunits; u += nwarps) {
    const uint32_t blk = u * 32u + lane;
    const bool valid = blk < p.nblocks;
    uint4 v[V];
#pragma unroll
    for (int k = 0; k < V; ++k) v[k] = make_uint4(0u, 0u, 0u, 0u);
    if (valid) {
      const uint32_t row = fdiv(blk, p.bpr);
      const uint16_t* src = p.x + (int64_t)row * p.ld + (int64_t)(blk - row * p.bpr.d) * (8 * V);
#pragma unroll
      for (int k = 0; k < V; ++k) v[k] = ld_stream(src + 8 * k);
    }
    quantize_block<FMT, RND, HAD, SFMMA, DQ>(p, v, blk, valid, lane, nv);
  }
}

// ======================================= TMA-fed axis-1 quantize / amax ===
// Contiguous inputs stream through a ring of 64 KB shared-memory stages filled
// by the bulk-copy engine: one producer thread issues a cp.async.bulk per stage
// (no per-thread load traffic, many bytes in flight), 15 to 31 consumer warps
// quantize (or reduce) each stage and release it through an mbarrier.
constexpr int kStreamChunks = 4096;                     // 8-element chunks per stage (64 KB of bf16)
constexpr int kStreamStages = 3;
constexpr int kStreamSmem = kStreamStages * kStreamChunks * 16 + 2 * kStreamStages * 8;
// Consumer warps per CTA (measured): 31 for NVFP4 and the amax (with the
// producer, the 1024-thread maximum, so at most 64 registers a thread, which
// their 16-element blocks fit); 16 for MXFP4 round-to-nearest, with or
// without rotation (31 warps ran 10-20 % slower, 19 warps at the same 96
// registers 5-6 % slower; for rotations of 64 and 128 elements, two blocks a
// thread on 15 warps, which keeps one or both cross-lane stages inside the
// thread, measured slower too: 20.1 -> 22.9 and 22.0 -> 24.1 us at 8192 x 4096);
// 15 for MXFP4 stochastic
// rounding, whose 32-element blocks with their eight Philox blocks want about
// 124 registers; 15 for four-over-six NVFP4, whose second candidate scale and
// fp64 error sums do not fit in 64 registers; 23 for NVFP4 stochastic rounding
// without rotation or dequantized output, whose Philox words then get up to 80
// registers (4096 x 4096: 31.9 -> 30.2 us; with the fused dequantize 23 warps
// were slower, 35.4 -> 36.1 us, and 27 the same).  Units of a stage are dealt
// to the warps round-robin, starting one place further on each stage, so that
// counts that do not divide evenly still balance over a run.
template <int FMT, int RND, int HAD = 0, int DQ = 0>
struct StreamWarps {
  static constexpr int kWarps =
      FMT == FMT_NV ? (RND == RND_SR && HAD == 0 && DQ == 0 ? 23 : 31) : (FMT == FMT_NV46 || RND == RND_SR ? 15 : 16);
  static constexpr int kThreads = 32 * (kWarps + 1);
};
constexpr int kAmaxWarps = 31;

struct StreamRing {
  uint4* data;
  uint64_t* full;
  uint64_t* empty;
};

__device__ __forceinline__ StreamRing stream_ring(uint8_t* smem) {
  StreamRing r;
  r.data = reinterpret_cast<uint4*>(smem);
  r.full = reinterpret_cast<uint64_t*>(smem + kStreamStages * kStreamChunks * 16);
  r.empty = r.full + kStreamStages;
  return r;
}

__device__ __forceinline__ void stream_ring_init(const StreamRing& r, int consumer_warps) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStreamStages; ++s) {
      mbar_init(smem_addr(&r.full[s]), 1);
      mbar_init(smem_addr(&r.empty[s]), (uint32_t)consumer_warps);
    }
    mbar_init_fence();
  }
}

// The CTA's share of the chunk range: whole 512-chunk granules (4096 elements,
// so stage starts stay aligned to scale blocks, Hadamard blocks and warp
// units), split as evenly as the granules allow, so that every SM gets the same
// work within one granule instead of whole 64 KB stages dealt round-robin.
struct StreamRange {
  uint32_t lo, hi;
};
__device__ __forceinline__ StreamRange stream_range(uint32_t nchunks) {
  constexpr uint32_t kGranule = 512;
  const uint32_t ng = (nchunks + kGranule - 1) / kGranule;
  const uint32_t g0 = (uint32_t)(((unsigned long long)ng * blockIdx.x) / gridDim.x);
  const uint32_t g1 = (uint32_t)(((unsigned long long)ng * (blockIdx.x + 1u)) / gridDim.x);
  return {min(g0 * kGranule, nchunks), min(g1 * kGranule, nchunks)};
}

// Producer (one thread): stage the CTA's range into the ring, kStreamChunks at
// a time.  On an expired wait it flags the error, lets every copy it issued
// land, and stops.
__device__ void stream_produce(const StreamRing& r, const uint16_t* x, uint32_t nchunks, unsigned* error) {
  const StreamRange rg = stream_range(nchunks);
  uint32_t stage = 0, phase = 0, issued = 0, parity_bits = 0;
  for (uint32_t c0 = rg.lo; c0 < rg.hi; c0 += kStreamChunks) {
    if (!mbar_wait_bounded(smem_addr(&r.empty[stage]), phase ^ 1u)) {
      if (error != nullptr) atomicOr(error, 4u);
      for (int s = 0; s < kStreamStages; ++s)
        if (issued & (1u << s)) mbar_wait_bounded(smem_addr(&r.full[s]), (parity_bits >> s) & 1u);
      return;
    }
    const uint32_t n = min((uint32_t)kStreamChunks, rg.hi - c0);
    const uint32_t fb = smem_addr(&r.full[stage]);
    mbar_expect_tx(fb, n * 16u);
    bulk_g2s(smem_addr(r.data + (size_t)stage * kStreamChunks), x + (size_t)c0 * 8, n * 16u, fb);
    issued |= 1u << stage;
    parity_bits = (parity_bits & ~(1u << stage)) | (phase << stage);
    if (++stage == kStreamStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
}

template <int FMT, int RND, int HAD, bool SFMMA, int DQ = 0>
__global__ void __launch_bounds__(StreamWarps<FMT, RND, HAD, DQ>::kThreads, 1) quantize_stream_kernel(QRowParams p) {
  constexpr int kStreamWarps = StreamWarps<FMT, RND, HAD, DQ>::kWarps;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ double tabd[128];
  pdl_trigger();
  const StreamRing r = stream_ring(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  stream_ring_init(r, kStreamWarps);
  pdl_wait();
  if (SFMMA) sf_pad_zero(p, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
  NvConsts nv{1.0f, 1.0, tabd};
  if (FMT != FMT_MX) {
    nv = nv_consts<kNvPairs<FMT, RND, DQ>>(*p.ts, tabd);
    if (p.ts_copy_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *p.ts_copy_out = nv.s_t;
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) stream_produce(r, p.x, p.nchunks, p.error);
    return;
  }
  const int cw = warp - 1;
  const StreamRange rg = stream_range(p.nchunks);
  uint32_t stage = 0, phase = 0, j = 0;
  for (uint32_t c0 = rg.lo; c0 < rg.hi; c0 += kStreamChunks, ++j) {
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(smem_addr(&r.full[stage]), phase) ? 1 : 0;
    if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
      if (lane == 0 && p.error != nullptr) atomicOr(p.error, 4u);
      return;
    }
    const uint32_t n = min((uint32_t)kStreamChunks, rg.hi - c0);
    const uint4* src = r.data + (size_t)stage * kStreamChunks;
    constexpr int V = BlockShape<FMT>::V;
    constexpr uint32_t kUnits = kStreamChunks / (32 * V);                   // warp units per full stage
    const uint32_t first = ((uint32_t)cw + kStreamWarps - (j * kUnits) % kStreamWarps) % kStreamWarps;
    for (uint32_t u = first; u * 32u * V < n; u += kStreamWarps) {         // warp-uniform
      const uint32_t lb = u * 32u + lane;                                    // block within the stage
      const bool valid = lb * V < n;
      uint4 v[V];
      const uint32_t sw = chunk_swap<FMT, HAD>(lane);
#pragma unroll
      for (int k = 0; k < V; ++k) v[k] = valid ? src[lb * V + ((uint32_t)k ^ sw)] : make_uint4(0u, 0u, 0u, 0u);
      quantize_block<FMT, RND, HAD, SFMMA, DQ, true>(p, v, c0 / V + lb, valid, lane, nv, sw);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&r.empty[stage]));
    if (++stage == kStreamStages) {
      stage = 0;
      phase ^= 1u;
    }
  }
}

// The amax pass on the same ring (contiguous input).
template <int HAD>
__global__ void __launch_bounds__(32 * (kAmaxWarps + 1), 1) amax_stream_kernel(AmaxParams p, unsigned* error) {
  constexpr int kStreamWarps = kAmaxWarps;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint32_t wmax[kStreamWarps];
  __shared__ bool is_last;
  pdl_trigger();
  const StreamRing r = stream_ring(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  stream_ring_init(r, kStreamWarps);
  pdl_wait();
  __syncthreads();
  float m = 0.0f;
  if (warp == 0) {
    if (lane == 0) stream_produce(r, p.x, p.rows_x_cpr, error);
  } else {
    const int cw = warp - 1;
    const StreamRange rg = stream_range(p.rows_x_cpr);
    uint32_t stage = 0, phase = 0;
    for (uint32_t c0 = rg.lo; c0 < rg.hi; c0 += kStreamChunks) {
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(smem_addr(&r.full[stage]), phase) ? 1 : 0;
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
        if (lane == 0 && error != nullptr) atomicOr(error, 4u);
        break;
      }
      const uint32_t n = min((uint32_t)kStreamChunks, rg.hi - c0);
      const uint4* src = r.data + (size_t)stage * kStreamChunks;
#pragma unroll
      for (int k = 0; k < kStreamChunks / 32 / kStreamWarps; ++k) {
        const uint32_t lt = (uint32_t)(cw + k * kStreamWarps);
        if (lt * 32u >= n) break;
        const uint32_t local = lt * 32u + lane;
        const uint4 v = local < n ? src[local] : make_uint4(0u, 0u, 0u, 0u);
        float x[8];
        unpack8(v, x);
        if (HAD) hadamard_rotate<HAD>(x, lane);
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(x[j]));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&r.empty[stage]));
      if (++stage == kStreamStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    const uint32_t b = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m));
    if (lane == 0) wmax[cw] = b;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int w = 0; w < kStreamWarps; ++w) b = max(b, wmax[w]);
    p.partials[blockIdx.x] = __uint_as_float(b);
    __threadfence();
    is_last = (atomicAdd(p.counter, 1u) == gridDim.x - 1);
  }
  __syncthreads();
  if (!is_last || warp != 0) return;
  uint32_t b = 0;
  for (uint32_t i = lane; i < gridDim.x; i += 32u) b = max(b, __float_as_uint(__ldcg(p.partials + i)));
  b = __reduce_max_sync(0xFFFFFFFFu, b);
  if (lane == 0) {
    const float amax = __uint_as_float(b);
    *p.out = p.mode == 0 ? amax : (amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f));
    *p.counter = 0u;
  }
}

// ============================================ single-pass NVFP4 quantize ===
// NVFP4 needs the tensor amax before any block can be scaled.  When the whole
// tensor fits in shared memory across the SMs (148 x ~227 KB on B200), one
// cooperative launch reads it from HBM once: each CTA stages a contiguous run
// of warp tiles in shared memory while reducing its amax, the CTAs meet at a
// bounded grid barrier, and each quantizes its staged slice.  Small tensors
// still take one 512-byte tile a CTA: a single CTA for a decode-sized
// activation (1 x 4096, tensor-core scale layout) measured 6.7 against 4.8 us,
// mostly the padding of the 128-row scale tiles written from one SM.
struct FusedParams {
  QRowParams q;
  float* ts_out;          // s_t, written by CTA 0
  float* partials;        // one partial amax per CTA
  unsigned* arrive;       // grid-barrier arrivals (zero at launch: the previous launch reset it)
  unsigned* depart;       // grid-barrier departures
  unsigned* error;        // device error word (bit 1: barrier wait expired)
  uint32_t tiles_per_cta; // 32-chunk warp tiles staged by each CTA
};

// Consumer warps: 31 (1024 threads in all, 64 registers a thread) for NVFP4; 15 for four-over-six,
// whose two candidate scales need about 100 registers.
template <int FMT>
struct FusedWarps {
  static constexpr int kWarps = FMT == FMT_NV46 ? 15 : 31;
  static constexpr int kThreads = 32 * (kWarps + 1);
};
constexpr int kFusedMaxSmem = 227 * 1024 - 2048;          // staged slice; room left for the static data
constexpr int kFusedPieces = 8;                           // bulk copies (and mbarriers) per slice

template <int FMT, int RND, int HAD, bool SFMMA, int DQ = 0>
__global__ void __launch_bounds__(FusedWarps<FMT>::kThreads, 1) nv_quantize_fused_kernel(FusedParams fp) {
  constexpr int kFusedWarps = FusedWarps<FMT>::kWarps;
  extern __shared__ __align__(1024) uint4 slice[];
  __shared__ double tabd[128];
  __shared__ float red[kFusedWarps];
  __shared__ float s_t_shared;
  __shared__ __align__(8) uint64_t piece_bar[kFusedPieces];
  const QRowParams& p = fp.q;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t ntiles = (p.nchunks + 31u) >> 5;
  const uint32_t t_begin = blockIdx.x * fp.tiles_per_cta;
  const uint32_t t_end = min(ntiles, t_begin + fp.tiles_per_cta);
  const uint32_t c_begin = t_begin * 32u;
  const uint32_t c_end = min(p.nchunks, t_end * 32u);
  const uint32_t nslice = c_end > c_begin ? c_end - c_begin : 0u;
  const uint32_t piece = ((nslice + kFusedPieces - 1) / kFusedPieces + 31u) & ~31u;   // chunks, whole warp tiles
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int k = 0; k < kFusedPieces; ++k) mbar_init(smem_addr(&piece_bar[k]), 1);
    mbar_init_fence();
  }
  pdl_wait();
  if (SFMMA) sf_pad_zero(p, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
  __syncthreads();
  // phase 1: the slice lands in shared memory as kFusedPieces bulk copies; consumers reduce the
  // amax (of the rotated values when HAD > 0) of each piece as soon as it arrives
  if (warp == 0) {
    if (lane == 0) {
      for (int k = 0; k < kFusedPieces; ++k) {
        const uint32_t a = min(nslice, (uint32_t)k * piece), b = min(nslice, (uint32_t)(k + 1) * piece);
        const uint32_t bar = smem_addr(&piece_bar[k]);
        if (b > a) {
          mbar_expect_tx(bar, (b - a) * 16u);
          bulk_g2s(smem_addr(slice + a), p.x + (size_t)(c_begin + a) * 8, (b - a) * 16u, bar);
        } else {
          mbar_arrive(bar);                                  // empty piece: complete its phase
        }
      }
    }
  } else {
    const int cw = warp - 1;
    float m = 0.0f;
    for (int k = 0; k < kFusedPieces; ++k) {
      const uint32_t a = min(nslice, (uint32_t)k * piece), b = min(nslice, (uint32_t)(k + 1) * piece);
      if (b <= a) continue;
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(smem_addr(&piece_bar[k]), 0u) ? 1 : 0;
      if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
        if (lane == 0) atomicOr(fp.error, 4u);
        break;
      }
      for (uint32_t lt = a / 32u + cw; lt * 32u < b; lt += kFusedWarps) {
        const uint32_t local = lt * 32u + lane;
        const uint4 v = local < b ? slice[local] : make_uint4(0u, 0u, 0u, 0u);
        float x[8];
        unpack8(v, x);
        if (HAD) hadamard_rotate<HAD>(x, lane);
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(x[j]));
      }
    }
    m = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m)));
    if (lane == 0) red[cw] = m;
  }
  __syncthreads();

  // grid barrier: publish this CTA's maximum, wait (bounded) for every CTA
  if (threadIdx.x == 0) {
    float cm = 0.0f;
    for (int w = 0; w < kFusedWarps; ++w) cm = fmaxf(cm, red[w]);
    fp.partials[blockIdx.x] = cm;
    __threadfence();
    atomicAdd(fp.arrive, 1u);
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
      unsigned n;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(n) : "l"(fp.arrive) : "memory");
      if (n >= gridDim.x) break;
      if (globaltimer_ns() - t0 > 2000000000ull) {       // 2 s: give up, flag the error, finish anyway
        atomicOr(fp.error, 2u);
        break;
      }
      __nanosleep(64);
    }
    // the last CTA to leave zeroes both counters for the next launch (every CTA has seen the
    // full count by then)
    if (atomicAdd(fp.depart, 1u) == gridDim.x - 1u) {
      atomicExch(fp.arrive, 0u);
      atomicExch(fp.depart, 0u);
    }
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t b = 0u;
    for (uint32_t i = lane; i < gridDim.x; i += 32u) b = max(b, __float_as_uint(__ldcg(fp.partials + i)));
    b = __reduce_max_sync(0xFFFFFFFFu, b);
    if (lane == 0) {
      const float amax = __uint_as_float(b);
      const float s_t = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
      s_t_shared = s_t;
      if (blockIdx.x == 0) *fp.ts_out = s_t;
    }
  }
  __syncthreads();
  const NvConsts nv = nv_consts<kNvPairs<FMT, RND, DQ>>(s_t_shared, tabd);
  __syncthreads();

  // phase 2: quantize the staged slice, one thread per 16-element block, on every warp (the
  // producer warp too: 4096^2 quantize + dequantize 24.7 -> 23.9 us, graph-replayed)
  for (uint32_t u = (uint32_t)warp; u * 64u < nslice; u += kFusedWarps + 1) {
    const uint32_t lb = u * 32u + lane;
    const bool valid = lb * 2u < nslice;
    uint4 v[2];
    const uint32_t sw = chunk_swap<FMT, HAD>(lane);
    v[0] = valid ? slice[lb * 2u + sw] : make_uint4(0u, 0u, 0u, 0u);
    v[1] = valid ? slice[lb * 2u + (sw ^ 1u)] : make_uint4(0u, 0u, 0u, 0u);
    quantize_block<FMT, RND, HAD, SFMMA, DQ, true>(p, v, c_begin / 2u + lb, valid, lane, nv, sw);
  }
}

// ======================================================== axis-0 quantize ===
// 4 x 4 transpose of 32-bit words across the four lanes of a quad: on entry lane q holds row q
// (w[0..3], one word per column); on return t[s] is word q of row s.  Two butterfly stages: with
// lane q ^ 1 swap the two words of the columns whose bit 0 differs from q's, then with lane q ^ 2
// the two (of four held) whose bit 1 differs; lane q then holds column q of rows q, q ^ 1, q ^ 2,
// q ^ 3, which two conditional swaps put in row order.  Every lane of the warp must call it.
__device__ __forceinline__ void quad_transpose4(const uint32_t (&w)[4], uint32_t (&t)[4], int lane) {
  const bool b0 = (lane & 1) != 0, b1 = (lane & 2) != 0;
  const uint32_t o0 = b0 ? w[1] : w[0], o1 = b0 ? w[3] : w[2];            // own columns with bit 0 = q0
  const uint32_t r0 = __shfl_xor_sync(0xFFFFFFFFu, b0 ? w[0] : w[1], 1);  // row q ^ 1, columns q0, 2 + q0
  const uint32_t r1 = __shfl_xor_sync(0xFFFFFFFFu, b0 ? w[2] : w[3], 1);
  const uint32_t a0 = b1 ? o1 : o0, a1 = b1 ? r1 : r0;                     // column q of rows q, q ^ 1
  const uint32_t a2 = __shfl_xor_sync(0xFFFFFFFFu, b1 ? o0 : o1, 2);      // column q of row q ^ 2
  const uint32_t a3 = __shfl_xor_sync(0xFFFFFFFFu, b1 ? r0 : r1, 2);      // column q of row q ^ 3
  // t[s] = a[s ^ q]
  const uint32_t u0 = b0 ? a1 : a0, u1 = b0 ? a0 : a1, u2 = b0 ? a3 : a2, u3 = b0 ? a2 : a3;
  t[0] = b1 ? u2 : u0;
  t[1] = b1 ? u3 : u1;
  t[2] = b1 ? u0 : u2;
  t[3] = b1 ? u1 : u3;
}

// Blocks run down the columns of x[R, C]; the output is written transposed
// (codes [C, R/2]).  A CTA stages a 128-row x 64-column bf16 tile in shared
// memory with coalesced 128-bit loads; each thread then owns one column and a
// 32-row segment (one MX block / two NV blocks) and writes its packed codes
// as one contiguous run of the output row.  For stochastic rounding the four
// lanes of a quad hold four adjacent columns (C is a multiple of 8), which
// share one Philox counter per row: each lane draws the block of one row and
// a quad transpose hands every lane its column's word, one Philox4x32-10
// evaluation per four elements as on axis 1.
struct QColParams {
  const uint16_t* x;
  uint32_t R, C;
  int64_t ld;
  uint32_t G, g4;        // k-groups per output row (R / block) and padded/4
  unsigned long long seed;
  PhiloxKeys keys;      // the seed's Philox key schedule
  unsigned long long jbase;  // Philox counter of element (0, 0) (row shards: first_row * C / 4)
  uint32_t mx_thr;      // MXFP4 exponent clip threshold (significand field; kMxClipOcp: the OCP rule)
  const float* ts;
  float* ts_copy_out;
  uint8_t* codes;
  uint8_t* scales;
};

template <int FMT, int RND, bool SFMMA>
__global__ void __launch_bounds__(256, (RND == RND_SR && FMT != FMT_NV46) ? 3 : 2) quantize_cols_kernel(QColParams p) {
  pdl_trigger();
  __shared__ __align__(16) uint16_t tile[128][64];
  __shared__ double tabd[128];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  const uint32_t tiles_r = (p.R + 127u) / 128u, tiles_c = (p.C + 63u) / 64u;
  NvConsts nv{1.0f, 1.0, tabd};
  if (FMT != FMT_MX) {
    nv = nv_consts(*p.ts, tabd);            // visible after the first __syncthreads of the tile loop
    if (p.ts_copy_out != nullptr && blockIdx.x == 0 && tid == 0) *p.ts_copy_out = nv.s_t;
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
    if (rbase >= p.R) continue;                  // warp-uniform; lanes past C stay for the shuffles
    const bool col_ok = c < p.C;
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
      float inv = 1.0f;
      double yd = 1.0;
      if (FMT == FMT_MX) {
        byte = mx_scale_byte_clip(am, p.mx_thr);
        inv = mx_inv_scale(byte);
        zero = (am == 0.0f);
      } else {
        byte = e4m3_rn_sat(nv_scale_arg64(am, nv.s_t, nv.yd_st));
        if (FMT == FMT_NV46) {
          float xb[BS];
#pragma unroll
          for (int i = 0; i < BS; ++i) xb[i] = xv[b * BS + i];
          byte = nv_four_over_six<RND, BS>(xb, am, byte, nv);
#pragma unroll
          for (int i = 0; i < BS; ++i) xv[b * BS + i] = xb[i];     // quotients under the chosen scale
        } else {
          yd = nv.tabd[byte];
        }
        zero = (byte == 0u);
      }
#pragma unroll
      for (int w8 = 0; w8 < BS / 8; ++w8) {
        float v8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xi = xv[b * BS + w8 * 8 + i];
          if (FMT == FMT_MX) {
            v8[i] = __fmul_rn(xi, inv);
          } else if (FMT == FMT_NV46) {
            v8[i] = xi;
          } else {
            v8[i] = div_by_recip64(xi, yd);
          }
        }
        uint32_t packed;
        if (RND == RND_RTN) {
          packed = pack8_rtn(v8);
        } else {
          // rows rb + 8*w8 + 4h + q (q = lane & 3): word (c & 3) of row i's block goes to element i
          uint32_t rw[8];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const unsigned long long row = rb + w8 * 8 + 4 * h + (lane & 3);
            const unsigned long long j = p.jbase + ((row * p.C + (c & ~3u)) >> 2);
            const u32x4 ph = philox4x32_10((uint32_t)j, (uint32_t)(j >> 32), p.keys);
            const uint32_t w[4] = {ph.x, ph.y, ph.z, ph.w};
            uint32_t t[4];
            quad_transpose4(w, t, lane);
#pragma unroll
            for (int i = 0; i < 4; ++i) rw[4 * h + i] = t[i];
          }
          uint32_t n[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) n[i] = e2m1_sr(v8[i], rw[i]);
          packed = pack8_nibbles(n);
        }
        words[b * (BS / 8) + w8] = zero ? 0u : packed;
      }
      if (!col_ok) continue;
      const uint32_t g = rb / BS;
      if (SFMMA) p.scales[sf_mma_offset(c, g, p.g4)] = (uint8_t)byte;
      else p.scales[(size_t)c * p.G + g] = (uint8_t)byte;
      if (FMT != FMT_MX) {
        *reinterpret_cast<uint2*>(p.codes + (size_t)c * (p.R / 2) + rb / 2) = make_uint2(words[2 * b], words[2 * b + 1]);
      }
    }
    if (FMT == FMT_MX && col_ok) {
      *reinterpret_cast<uint4*>(p.codes + (size_t)c * (p.R / 2) + rbase / 2) =
          make_uint4(words[0], words[1], words[2], words[3]);
    }
  }
}

// MXFP4 stochastic rounding along axis 0 with four adjacent columns and eight rows a thread: the
// four columns share one Philox4x32-10 evaluation per row (counter (row * C + c) / 4 for c a
// multiple of 4, word c & 3), so every word is drawn where it is used, with no exchange between
// lanes (the kernel above hands each lane its column's words through a quad transpose per four
// rows).  A quad's lanes hold the four 8-row slices of the same four columns, one 32-row block
// each: a two-stage shuffle gives the blocks' maxima, and one quad transpose of the packed codes
// (one 32-bit word per column and slice) lets lane q store column q's 16 bytes of codes.  The
// 128 x 64 bf16 tile's 16-byte chunks sit XOR-ed with bit 3 of the row moved to chunk bit 2, so
// that the four 8-row slices of a warp's 8-byte reads fall in two bank halves.
template <bool SFMMA>
__global__ void __launch_bounds__(256, 4) quantize_cols_mx_sr_kernel(QColParams p) {
  pdl_trigger();
  __shared__ __align__(16) uint16_t tile[128][64];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = warp & 1, seg = warp >> 1, cgi = lane >> 2, rgi = lane & 3;
  pdl_wait();
  const uint32_t tiles_r = (p.R + 127u) / 128u, tiles_c = (p.C + 63u) / 64u;
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
      *reinterpret_cast<uint4*>(&tile[row][(ch ^ (((row >> 3) & 1) << 2)) * 8]) = v;
    }
    __syncthreads();
    const uint32_t rbase = r0 + 32u * seg;                   // the warp's 32 rows: one block per column
    if (rbase >= p.R) continue;                               // warp-uniform (R is a multiple of 32)
    const uint32_t cq = c0 + 32u * half + 4u * cgi;           // the lane's first column (a multiple of 4)
    float x[8][4];
    const int colt = 32 * half + 4 * cgi;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = 32 * seg + 8 * rgi + i;
      const int phys = (((colt >> 3) ^ (((row >> 3) & 1) << 2)) << 3) + (colt & 7);
      const uint2 w = *reinterpret_cast<const uint2*>(&tile[row][phys]);
      x[i][0] = bf16_lo(w.x); x[i][1] = bf16_hi(w.x);
      x[i][2] = bf16_lo(w.y); x[i][3] = bf16_hi(w.y);
    }
    float am[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i][k]));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      am[k] = m;
    }
    uint32_t byte[4];
    float inv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      byte[k] = mx_scale_byte_clip(am[k], p.mx_thr);
      inv[k] = mx_inv_scale(byte[k]);
    }
    uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const unsigned long long row = rbase + 8u * rgi + i;
      const unsigned long long j = p.jbase + ((row * p.C + cq) >> 2);
      const u32x4 ph = philox4x32_10((uint32_t)j, (uint32_t)(j >> 32), p.keys);
      const uint32_t r4[4] = {ph.x, ph.y, ph.z, ph.w};
      const float2 v01 = mul2(make_float2(x[i][0], x[i][1]), make_float2(inv[0], inv[1]));   // exact scaling
      const float2 v23 = mul2(make_float2(x[i][2], x[i][3]), make_float2(inv[2], inv[3]));
      words[0] |= e2m1_sr(v01.x, r4[0]) << (4 * i);
      words[1] |= e2m1_sr(v01.y, r4[1]) << (4 * i);
      words[2] |= e2m1_sr(v23.x, r4[2]) << (4 * i);
      words[3] |= e2m1_sr(v23.y, r4[3]) << (4 * i);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) words[k] = am[k] == 0.0f ? 0u : words[k];
    uint32_t t4[4];
    quad_transpose4(words, t4, lane);                         // t4[s]: column cq + rgi, rows 8s .. 8s + 7
    const uint32_t c = cq + (uint32_t)rgi;
    if (c >= p.C) continue;
    *reinterpret_cast<uint4*>(p.codes + (size_t)c * (p.R / 2) + rbase / 2) = make_uint4(t4[0], t4[1], t4[2], t4[3]);
    const uint32_t b = rgi == 0 ? byte[0] : rgi == 1 ? byte[1] : rgi == 2 ? byte[2] : byte[3];
    const uint32_t g = rbase / 32u;
    if (SFMMA) p.scales[sf_mma_offset(c, g, p.g4)] = (uint8_t)b;
    else p.scales[(size_t)c * p.G + g] = (uint8_t)b;
  }
}

// ===================================================== 2-D (square-tile) quantize ===
// "Pretraining Large Language Models with NVFP4", Abstract: a two-dimensional
// scheme gives weights one consistent representation forward and backward.
// A block x block tile (16 x 16 NVFP4, 32 x 32 MXFP4) shares one scale; every
// element is scaled and rounded once, and its code goes both to W's codes
// (packed along rows, [R, C/2]) and, when asked, to W^T's codes (packed along
// W's columns, [C, R/2]), each row or column segment carrying the tile's
// scale byte.  A CTA takes (4 x block) x 64 tiles of W; thread t owns the row
// segment (row t % (4 block), block columns of segment t / (4 block)), so the
// `block` rows of a square tile sit on consecutive lanes: the tile amax is a
// shuffle reduction, and each row segment is quantized like a 1-D block (same
// Philox indices).  Tiles arrive in shared memory by coalesced 16-byte async
// copies (8 lanes per 128-byte row; the next tile's in flight while the
// current one is processed), their 16-byte chunks XOR-swizzled by row so that
// the lanes' row-segment reads are conflict-free.  W's codes
// leave as the packed words of each row; W^T's come from 8 x 8 nibble
// transposes across groups of 8 lanes (three shuffle stages), and both are
// gathered in shared memory so that one thread writes a whole output row
// segment (32 bytes of W, 32 or 64 bytes of W^T) with sector-wide stores.
struct Q2Params {
  const uint16_t* x;
  uint32_t R, C;
  int64_t ld;
  unsigned long long seed;
  PhiloxKeys keys;      // the seed's Philox key schedule
  uint32_t mx_thr;      // MXFP4 exponent clip threshold (significand field; kMxClipOcp: the OCP rule)
  const float* ts;
  float* ts_copy_out;
  uint8_t* codes;        // [R, C/2]
  uint8_t* scales;       // [R, C/bs] or tensor-core layout (R rows, C/bs groups)
  uint8_t* codes_t;      // [C, R/2] or null
  uint8_t* scales_t;     // [C, R/bs] or tensor-core layout (C rows, R/bs groups)
  uint32_t g4, g4_t;     // padded groups / 4 of the two scale tensors (tensor-core layout)
};

// Transpose of the 8 x 8 nibble matrix held by the 8 lanes of an aligned lane group (lane j: row
// j, nibble i = column i): on return lane i holds column i (nibble j = row j).  Every lane of the
// warp must call it.
__device__ __forceinline__ uint32_t nibble_transpose8(uint32_t v, int lane) {
  uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, v, 4);
  v = (lane & 4) ? ((v & 0xFFFF0000u) | (o >> 16)) : ((v & 0x0000FFFFu) | (o << 16));
  o = __shfl_xor_sync(0xFFFFFFFFu, v, 2);
  v = (lane & 2) ? ((v & 0xFF00FF00u) | ((o & 0xFF00FF00u) >> 8)) : ((v & 0x00FF00FFu) | ((o & 0x00FF00FFu) << 8));
  o = __shfl_xor_sync(0xFFFFFFFFu, v, 1);
  v = (lane & 1) ? ((v & 0xF0F0F0F0u) | ((o & 0xF0F0F0F0u) >> 4)) : ((v & 0x0F0F0F0Fu) | ((o & 0x0F0F0F0Fu) << 4));
  return v;
}

// N bytes of words (N = 32 or 64) to dst, of which the first n (a multiple of 8) are written:
// 32-byte stores (mode 32: dst 32-byte aligned and n == N), 16-byte (mode 16) or 8-byte stores.
template <int N>
__device__ __forceinline__ void store_segment(uint8_t* dst, const uint32_t (&w)[N / 4], uint32_t n, int mode) {
  if (n == N && mode == 32) {
#pragma unroll
    for (int k = 0; k < N / 32; ++k)
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 32 * k), "r"(w[8 * k]),
                   "r"(w[8 * k + 1]), "r"(w[8 * k + 2]), "r"(w[8 * k + 3]), "r"(w[8 * k + 4]), "r"(w[8 * k + 5]),
                   "r"(w[8 * k + 6]), "r"(w[8 * k + 7])
                   : "memory");
  } else if (n == N && mode == 16) {
#pragma unroll
    for (int k = 0; k < N / 16; ++k)
      reinterpret_cast<uint4*>(dst)[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  } else {
#pragma unroll
    for (int k = 0; k < N / 8; ++k)
      if (8u * k < n) reinterpret_cast<uint2*>(dst)[k] = make_uint2(w[2 * k], w[2 * k + 1]);
  }
}

template <int FMT, int RND, bool SFMMA>
__global__ void __launch_bounds__(256) quantize_2d_kernel(Q2Params p) {
  pdl_trigger();
  constexpr int BS = FMT == FMT_MX ? 32 : 16;
  constexpr int TR = 4 * BS, TC = 64;                     // CTA tile: (4 x block) rows x 64 columns
  constexpr int SEGS = TC / BS;                           // row segments (square tiles) across the CTA tile
  constexpr int V = BS / 8;                               // 16-byte chunks (and code words) per segment
  constexpr int RG = TR / 8;                              // 8-row groups
  constexpr int ROWW = TC / 8 + 1;                        // W words per row (+1: conflict-free parking)
  constexpr int COLW = RG + 4;                             // W^T words per column (+4: 16-byte rows, no conflicts)
  __shared__ __align__(16) uint4 xin[2][TR * 8];       // two input tiles: row r, chunk j at r * 8 + (j ^ r % 8)
  __shared__ uint32_t code_row[TR * ROWW];
  __shared__ __align__(16) uint32_t code_col[TC * COLW];
  __shared__ uint8_t sc_row[TR][SEGS];
  __shared__ uint8_t sc_col[TC][4];
  __shared__ double tabd[128];
  const int tid = threadIdx.x, lane = tid & 31;
  const int row = tid % TR, seg = tid / TR;
  pdl_wait();
  NvConsts nv{1.0f, 1.0, tabd};
  if (FMT != FMT_MX) {
    nv = nv_consts(*p.ts, tabd);
    if (p.ts_copy_out != nullptr && blockIdx.x == 0 && tid == 0) *p.ts_copy_out = nv.s_t;
  }
  __syncthreads();                                        // the scale table is read by the first tile
  // store widths of the two outputs (rows of W's codes are C/2 bytes apart, of W^T's R/2)
  auto mode_of = [](const void* base, uint32_t pitch) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(base);
    return (a % 32 == 0 && pitch % 32 == 0) ? 32 : (a % 16 == 0 && pitch % 16 == 0) ? 16 : 8;
  };
  const int mode_w = mode_of(p.codes, p.C / 2);
  const int mode_t = p.codes_t != nullptr ? mode_of(p.codes_t, p.R / 2) : 8;
  const uint32_t tiles_r = (p.R + TR - 1) / TR, tiles_c = (p.C + TC - 1) / TC;
  const uint32_t ntiles = tiles_r * tiles_c;
  // async copies of tile t into buffer b: thread i moves chunks i, i + 256, ... (row q / 8,
  // chunk q % 8); chunks outside the matrix are zero-filled
  auto issue = [&](uint32_t t, int b) {
    if (t < ntiles) {
      const uint32_t r0 = (t / tiles_c) * TR, c0 = (t % tiles_c) * TC;
#pragma unroll
      for (int q = tid; q < TR * 8; q += 256) {
        const uint32_t r = (uint32_t)q / 8u, j = (uint32_t)q % 8u;
        const uint32_t gr = r0 + r, gc = c0 + 8u * j;
        const uint32_t dst = smem_addr(&xin[b][r * 8 + (j ^ (r % 8u))]);
        const bool in = gr < p.R && gc < p.C;
        const uint16_t* src = in ? p.x + (int64_t)gr * p.ld + gc : p.x;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(in ? 16 : 0)
                     : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  issue(blockIdx.x, 0);
  int buf = 0;
  for (uint32_t t = blockIdx.x; t < ntiles; t += gridDim.x, buf ^= 1) {
    issue(t + gridDim.x, buf ^ 1);                        // in flight while this tile is processed
    asm volatile("cp.async.wait_group 1;" ::: "memory");  // this tile's copies have landed
    __syncthreads();
    const uint32_t r0 = (t / tiles_c) * TR, c0 = (t % tiles_c) * TC;
    const uint32_t grow = r0 + row, gcol = c0 + seg * BS;
    float x[BS];
#pragma unroll
    for (int k = 0; k < V; ++k) {
      const uint32_t j = (uint32_t)(seg * V + k);
      float t8[8];
      unpack8(xin[buf][row * 8 + (j ^ ((uint32_t)row % 8u))], t8);
#pragma unroll
      for (int i = 0; i < 8; ++i) x[8 * k + i] = t8[i];
    }
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < BS; ++i) am = fmaxf(am, fabsf(x[i]));
#pragma unroll
    for (int off = BS / 2; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, off));
    uint32_t byte;
    bool zero;
    if (FMT == FMT_MX) {
      byte = mx_scale_byte_clip(am, p.mx_thr);
      const float inv = mx_inv_scale(byte);
#pragma unroll
      for (int i = 0; i < BS; ++i) x[i] = __fmul_rn(x[i], inv);
      zero = (am == 0.0f);
    } else {
      byte = e4m3_rn_sat(nv_scale_arg64(am, nv.s_t, nv.yd_st));
      zero = (byte == 0u);
      nv_divide_block64<BS>(x, nv.tabd[byte], x);
    }
    uint32_t w[V];
    if (RND == RND_RTN) {
#pragma unroll
      for (int k = 0; k < V; ++k)
        w[k] = e2m1x4_rn(x[8 * k], x[8 * k + 1], x[8 * k + 2], x[8 * k + 3], x[8 * k + 4], x[8 * k + 5], x[8 * k + 6],
                         x[8 * k + 7]);
    } else {
      const unsigned long long j0 = ((unsigned long long)grow * p.C + gcol) >> 2;   // gcol % 4 == 0
#pragma unroll
      for (int k = 0; k < V; ++k) {
        const unsigned long long j = j0 + 2u * k;
        const u32x4 a = philox4x32_10((uint32_t)j, (uint32_t)(j >> 32), p.keys);
        const u32x4 b = philox4x32_10((uint32_t)(j + 1), (uint32_t)((j + 1) >> 32), p.keys);
        const float* xe = x + 8 * k;
        const uint32_t n[8] = {e2m1_sr(xe[0], a.x), e2m1_sr(xe[1], a.y), e2m1_sr(xe[2], a.z), e2m1_sr(xe[3], a.w),
                               e2m1_sr(xe[4], b.x), e2m1_sr(xe[5], b.y), e2m1_sr(xe[6], b.z), e2m1_sr(xe[7], b.w)};
        w[k] = pack8_nibbles(n);
      }
    }
    if (zero) {
#pragma unroll
      for (int k = 0; k < V; ++k) w[k] = 0u;
    }
    uint32_t wt[V];
#pragma unroll
    for (int k = 0; k < V; ++k) wt[k] = nibble_transpose8(w[k], lane);   // column 8k + lane % 8, 8 rows
    __syncthreads();                                      // the previous tile's write-out read its data
#pragma unroll
    for (int k = 0; k < V; ++k) {
      code_row[row * ROWW + seg * V + k] = w[k];
      code_col[(seg * BS + 8 * k + (lane & 7)) * COLW + row / 8] = wt[k];
    }
    sc_col[seg * BS + row % BS][row / BS] = (uint8_t)byte;
    sc_row[row][seg] = (uint8_t)byte;
    __syncthreads();
    const uint32_t vcols = min((uint32_t)TC, p.C > c0 ? p.C - c0 : 0u);      // multiples of the block
    const uint32_t vrows = min((uint32_t)TR, p.R > r0 ? p.R - r0 : 0u);
    if (tid < TR) {
      const uint32_t lr = (uint32_t)tid;
      if (lr < vrows) {
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = code_row[lr * ROWW + k];
        store_segment<32>(p.codes + (size_t)(r0 + lr) * (p.C / 2) + c0 / 2, o, vcols / 2, mode_w);
#pragma unroll
        for (int g = 0; g < SEGS; ++g) {
          if ((uint32_t)(g * BS) >= vcols) break;
          const uint32_t gg = c0 / BS + g;
          if (SFMMA) p.scales[sf_mma_offset(r0 + lr, gg, p.g4)] = sc_row[lr][g];
          else p.scales[(size_t)(r0 + lr) * (p.C / BS) + gg] = sc_row[lr][g];
        }
      }
    } else if (p.codes_t != nullptr && tid < TR + TC) {
      const uint32_t lc = (uint32_t)(tid - TR);
      if (lc < vcols) {
        uint32_t o[RG];
#pragma unroll
        for (int k = 0; k < RG / 4; ++k) {
          const uint4 q = *reinterpret_cast<const uint4*>(&code_col[lc * COLW + 4 * k]);
          o[4 * k] = q.x;
          o[4 * k + 1] = q.y;
          o[4 * k + 2] = q.z;
          o[4 * k + 3] = q.w;
        }
        store_segment<TR / 2>(p.codes_t + (size_t)(c0 + lc) * (p.R / 2) + r0 / 2, o, vrows / 2, mode_t);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          if ((uint32_t)(a * BS) >= vrows) break;
          const uint32_t gg = r0 / BS + a;
          if (SFMMA) p.scales_t[sf_mma_offset(c0 + lc, gg, p.g4_t)] = sc_col[lc][a];
          else p.scales_t[(size_t)(c0 + lc) * (p.R / BS) + gg] = sc_col[lc][a];
        }
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");   // no copy outlives the CTA
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

// Address of the scale byte of a chunk (8 codes) in either scale layout.
template <int FMT, bool SFMMA>
__device__ __forceinline__ const uint8_t* deq_scale_ptr(const DeqParams& p, uint32_t chunk) {
  constexpr int LPB = FMT == FMT_MX ? 4 : 2;             // chunks per scale block
  if (SFMMA) {
    const uint32_t row = fdiv(chunk, p.cpr);
    return p.scales + sf_mma_offset(row, (chunk - row * p.cpr.d) / LPB, p.g4);
  }
  return p.scales + chunk / LPB;
}

// One chunk of 8 codes to fp32 (or bf16) values.  NV: fp32(fp32(G[c] * sb) * s_t), where the
// product G[c] * sb (at most 6 significant bits, in [2^-10, 2688] or zero) is exact in f16.
// MX: G[c] * 2^E in fp32.
template <int FMT, bool BF16>
__device__ __forceinline__ void dequantize_chunk_to(const DeqParams& p, uint32_t byte, uint32_t slot, uint32_t w,
                                                    float s_t) {
  uint32_t h[4];
  e2m1x8_to_f16x2(w, h);
  float y[8];
  if (FMT == FMT_MX) {
    const float sc = mx_scale_value(byte);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 g = __half22float2(*reinterpret_cast<const __half2*>(&h[k]));
      const float2 r = mul2(g, splat2(sc));
      y[2 * k] = r.x;
      y[2 * k + 1] = r.y;
    }
  } else {
    const __half2 sb = __float2half2_rn(e4m3_value(byte));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 g = __half22float2(__hmul2(*reinterpret_cast<const __half2*>(&h[k]), sb));
      const float2 r = mul2(g, splat2(s_t));
      y[2 * k] = r.x;
      y[2 * k + 1] = r.y;
    }
  }
  if (BF16) {
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(y[2 * i]));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(y[2 * i + 1]));
      o[i] = lo | (hi << 16);
    }
    reinterpret_cast<uint4*>(p.out)[slot] = make_uint4(o[0], o[1], o[2], o[3]);
  } else {
    float4* o = reinterpret_cast<float4*>(p.out) + (size_t)slot * 2;
    o[0] = make_float4(y[0], y[1], y[2], y[3]);
    o[1] = make_float4(y[4], y[5], y[6], y[7]);
  }
}

// Dequantize with direct stores: consecutive threads own consecutive 8-code chunks, so each
// warp store covers 1 KB (fp32, one 32-byte store per lane when the output is 32-byte aligned) or
// 512 B (bf16) of contiguous output, whole L2 sectors; four chunks per thread per iteration have
// their code and scale loads in flight together.
constexpr int kDeqDirectUnroll = 4;

template <int FMT, bool SFMMA, bool BF16>
__global__ void __launch_bounds__(256) dequantize_direct_kernel(DeqParams p) {
  pdl_trigger();
  pdl_wait();
  const float s_t = FMT == FMT_NV ? *p.ts : 1.0f;
  const bool wide = !BF16 && (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t base = blockIdx.x * blockDim.x + threadIdx.x; base < p.nchunks;
       base += kDeqDirectUnroll * stride) {
    uint32_t w[kDeqDirectUnroll], b[kDeqDirectUnroll];
#pragma unroll
    for (int u = 0; u < kDeqDirectUnroll; ++u) {
      const uint32_t c = base + u * stride;
      w[u] = 0u;
      b[u] = 0u;
      if (c < p.nchunks) {
        w[u] = __ldg(p.codes + c);
        b[u] = __ldg(deq_scale_ptr<FMT, SFMMA>(p, c));
      }
    }
#pragma unroll
    for (int u = 0; u < kDeqDirectUnroll; ++u) {
      const uint32_t c = base + u * stride;
      if (c >= p.nchunks) break;
      uint32_t h[4];
      e2m1x8_to_f16x2(w[u], h);
      float y[8];
      const __half2 sb = __float2half2_rn(FMT == FMT_MX ? 1.0f : e4m3_value(b[u]));
      const float sc = FMT == FMT_MX ? mx_scale_value(b[u]) : s_t;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 hv = *reinterpret_cast<const __half2*>(&h[k]);
        const float2 g = __half22float2(FMT == FMT_MX ? hv : __hmul2(hv, sb));
        const float2 r = mul2(g, splat2(sc));
        y[2 * k] = r.x;
        y[2 * k + 1] = r.y;
      }
      if (BF16) {
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          o[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y[2 * i])) |
                 ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y[2 * i + 1])) << 16);
        reinterpret_cast<uint4*>(p.out)[c] = make_uint4(o[0], o[1], o[2], o[3]);
      } else if (wide) {
        float* o = static_cast<float*>(p.out) + (size_t)c * 8;
        asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(o), "f"(y[0]), "f"(y[1]),
                     "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7])
                     : "memory");
      } else {
        float4* o = reinterpret_cast<float4*>(p.out) + (size_t)c * 2;
        o[0] = make_float4(y[0], y[1], y[2], y[3]);
        o[1] = make_float4(y[4], y[5], y[6], y[7]);
      }
    }
  }
}

// Dequantize through shared memory: each CTA fills 512-chunk output tiles
// (16 KB fp32 / 8 KB bf16) in a 4-deep staging ring and writes each tile back
// with one bulk store, so the stores never queue behind per-thread traffic.
// A CTA owns a contiguous, evenly sized run of tiles, and the codes and scale
// bytes of the next three tiles are in flight while the current one is converted.
constexpr int kDeqTileChunks = 512;
constexpr int kDeqStages = 4;
constexpr int kDeqThreads = 256;

template <int FMT, bool SFMMA, bool BF16>
__global__ void __launch_bounds__(kDeqThreads) dequantize_stream_kernel(DeqParams p) {
  constexpr int kOut = BF16 ? 16 : 32;                   // output bytes per chunk
  constexpr int kTileBytes = kDeqTileChunks * kOut;
  extern __shared__ __align__(128) uint8_t stage_buf[];
  pdl_trigger();
  pdl_wait();
  const float s_t = FMT == FMT_NV ? *p.ts : 1.0f;
  const uint32_t ntiles = (p.nchunks + kDeqTileChunks - 1) / kDeqTileChunks;
  const uint32_t t0 = (uint32_t)(((unsigned long long)ntiles * blockIdx.x) / gridDim.x);
  const uint32_t t1 = (uint32_t)(((unsigned long long)ntiles * (blockIdx.x + 1u)) / gridDim.x);
  DeqParams q = p;
  // codes and scale bytes of the next kDeqAhead tiles are in flight while a tile is converted
  constexpr int kDeqAhead = 3;
  uint32_t wq[kDeqAhead][2], bq[kDeqAhead][2];
  auto fetch = [&](uint32_t tile, uint32_t (&w)[2], uint32_t (&b)[2]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t c = tile * kDeqTileChunks + threadIdx.x + k * kDeqThreads;
      w[k] = 0u;
      b[k] = 0u;
      if (tile < t1 && c < p.nchunks) {
        w[k] = __ldg(p.codes + c);
        b[k] = __ldg(deq_scale_ptr<FMT, SFMMA>(p, c));
      }
    }
  };
#pragma unroll
  for (int a = 0; a < kDeqAhead; ++a) fetch(t0 + (uint32_t)a, wq[a], bq[a]);
  int it = 0;
  for (uint32_t i = t0; i < t1; ++i, ++it) {
    const int stage = it % kDeqStages;
    const uint32_t w[2] = {wq[0][0], wq[0][1]}, sb[2] = {bq[0][0], bq[0][1]};
#pragma unroll
    for (int a = 0; a + 1 < kDeqAhead; ++a) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        wq[a][k] = wq[a + 1][k];
        bq[a][k] = bq[a + 1][k];
      }
    }
    fetch(i + (uint32_t)kDeqAhead, wq[kDeqAhead - 1], bq[kDeqAhead - 1]);
    if (threadIdx.x == 0 && it >= kDeqStages) bulk_wait_read<kDeqStages - 1>();
    __syncthreads();                                      // this stage's previous store has read its data
    q.out = stage_buf + stage * kTileBytes;               // chunk-local output pointer
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t local = threadIdx.x + k * kDeqThreads;
      const uint32_t c = i * kDeqTileChunks + local;
      if (c < p.nchunks) dequantize_chunk_to<FMT, BF16>(q, sb[k], local, w[k], s_t);
    }
    fence_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t n = min((uint32_t)kDeqTileChunks, p.nchunks - i * kDeqTileChunks);
      bulk_s2g(static_cast<uint8_t*>(p.out) + (size_t)i * kTileBytes, smem_addr(stage_buf + stage * kTileBytes),
               n * (uint32_t)kOut);
    }
  }
  if (threadIdx.x == 0) bulk_wait_all();
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
  return launch_kernel(amax_kernel<HAD>, dim3(grid), dim3(256), 0, st, false, 1u, ap);
}

template <int HAD>
static cudaError_t amax_stream_launch(const AmaxParams& ap, int num_sms, unsigned* error, cudaStream_t st) {
  static const cudaError_t attr =
      cudaFuncSetAttribute(amax_stream_kernel<HAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem);
  if (attr != cudaSuccess) return attr;
  const uint32_t ngran = (ap.rows_x_cpr + 511u) / 512u;      // stream_range's granules
  uint32_t grid = (uint32_t)num_sms;
  if (grid > (uint32_t)kMaxAmaxBlocks) grid = kMaxAmaxBlocks;
  if (ngran < grid) grid = ngran > 0 ? ngran : 1;
  return launch_kernel(amax_stream_kernel<HAD>, dim3(grid), dim3(32 * (kAmaxWarps + 1)), kStreamSmem, st, false, 1u,
                       ap, error);
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
  if (ap.contig) {
    switch (had) {
      case 0: return amax_stream_launch<0>(ap, num_sms, s.error, st);
      case 16: return amax_stream_launch<16>(ap, num_sms, s.error, st);
      case 32: return amax_stream_launch<32>(ap, num_sms, s.error, st);
      case 64: return amax_stream_launch<64>(ap, num_sms, s.error, st);
      case 128: return amax_stream_launch<128>(ap, num_sms, s.error, st);
      default: return cudaErrorInvalidValue;
    }
  }
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
  return launch_kernel(amax_kernel<0>, dim3(grid), dim3(256), 0, st, false, 1u, ap);
}

cudaError_t load_amax_fixed_grid_kernel() {
  cudaFuncAttributes a;
  return cudaFuncGetAttributes(&a, amax_kernel<0>);
}

cudaError_t launch_nv_tensor_scale(const float* amax, float* out, cudaStream_t st) {
  return launch_kernel(nv_tensor_scale_kernel, dim3(1), dim3(1), 0, st, false, 1u, amax, out);
}

template <int FMT, int RND, int HAD, bool SFMMA, int DQ = 0>
static cudaError_t rows_stream_launch(const QRowParams& qp, int num_sms, cudaStream_t st) {
  auto kernel = quantize_stream_kernel<FMT, RND, HAD, SFMMA, DQ>;
  static const cudaError_t attr =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStreamSmem);
  if (attr != cudaSuccess) return attr;
  const uint32_t ngran = (qp.nchunks + 511u) / 512u;         // stream_range's granules
  uint32_t grid = (uint32_t)num_sms;
  if (ngran < grid) grid = ngran > 0 ? ngran : 1;
  return launch_kernel(kernel, dim3(grid), dim3(StreamWarps<FMT, RND, HAD, DQ>::kThreads), kStreamSmem, st, false, 1u, qp);
}

template <int FMT, int RND, int HAD, bool SFMMA, int DQ = 0>
static cudaError_t rows_launch(const QRowParams& qp, int num_sms, cudaStream_t st) {
  if (qp.contig) return rows_stream_launch<FMT, RND, HAD, SFMMA, DQ>(qp, num_sms, st);
  static int occ = resident_ctas(quantize_rows_kernel<FMT, RND, HAD, SFMMA, DQ>, 256);
  const uint32_t nunits = (qp.nblocks + 31u) / 32u;
  uint32_t want = (nunits + 7u) / 8u;
  uint32_t grid = (uint32_t)num_sms * (uint32_t)occ;
  if (want < grid) grid = want > 0 ? want : 1;
  return launch_kernel(quantize_rows_kernel<FMT, RND, HAD, SFMMA, DQ>, dim3(grid), dim3(256), 0, st, false, 1u, qp);
}

template <int FMT, int RND, int HAD>
static cudaError_t rows_dispatch_sf(const QRowParams& qp, bool sfmma, int num_sms, cudaStream_t st) {
  return sfmma ? rows_launch<FMT, RND, HAD, true>(qp, num_sms, st) : rows_launch<FMT, RND, HAD, false>(qp, num_sms, st);
}

// Quantize + dequantize variants (no rotation): dq 1 = fp32 values, 2 = bf16.
template <int FMT, int RND>
static cudaError_t rows_dispatch_dq(const QRowParams& qp, int dq, bool sfmma, int num_sms, cudaStream_t st) {
  if (dq == 1)
    return sfmma ? rows_launch<FMT, RND, 0, true, 1>(qp, num_sms, st) : rows_launch<FMT, RND, 0, false, 1>(qp, num_sms, st);
  return sfmma ? rows_launch<FMT, RND, 0, true, 2>(qp, num_sms, st) : rows_launch<FMT, RND, 0, false, 2>(qp, num_sms, st);
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

template <int FMT, int RND, int HAD, bool SFMMA, int DQ = 0>
static cudaError_t fused_launch(const FusedParams& fp, uint32_t grid, size_t smem, cudaStream_t st) {
  auto kernel = nv_quantize_fused_kernel<FMT, RND, HAD, SFMMA, DQ>;
  static const cudaError_t attr =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedMaxSmem);
  if (attr != cudaSuccess) return attr;
  return launch_kernel(kernel, dim3(grid), dim3(FusedWarps<FMT>::kThreads), smem, st, true, 1u, fp);
}

template <int RND, int HAD, int FMT = FMT_NV>
static cudaError_t fused_dispatch_sf(const FusedParams& fp, bool sfmma, uint32_t grid, size_t smem, cudaStream_t st) {
  return sfmma ? fused_launch<FMT, RND, HAD, true>(fp, grid, smem, st)
               : fused_launch<FMT, RND, HAD, false>(fp, grid, smem, st);
}

bool fused_nv_fits(int64_t rows, int64_t cols, int num_sms, size_t* smem_out, uint32_t* tiles_per_cta) {
  const uint64_t nchunks = (uint64_t)rows * (uint64_t)(cols / 8);
  const uint64_t ntiles = (nchunks + 31u) / 32u;
  const uint64_t per = (ntiles + (uint64_t)num_sms - 1) / (uint64_t)num_sms;
  const size_t smem = (size_t)per * 32u * 16u;
  if (smem > (size_t)kFusedMaxSmem || num_sms > kMaxAmaxBlocks) return false;
  *smem_out = smem;
  *tiles_per_cta = (uint32_t)per;
  return true;
}

cudaError_t launch_quantize_nv_fused(const QuantizeParams& p, float* ts_out, const Scratch& s, int num_sms,
                                     cudaStream_t st) {
  size_t smem = 0;
  uint32_t per = 0;
  if (!fused_nv_fits(p.rows, p.cols, num_sms, &smem, &per)) return cudaErrorInvalidValue;
  FusedParams fp;
  QRowParams& qp = fp.q;
  qp.x = static_cast<const uint16_t*>(p.x);
  qp.nchunks = (uint32_t)(p.rows * (p.cols / 8));
  qp.nblocks = (uint32_t)(p.rows * (p.cols / 16));
  qp.bpr = make_fastdiv((uint32_t)(p.cols / 16));
  qp.cpr = make_fastdiv((uint32_t)(p.cols / 8));
  qp.ld = p.ld;
  qp.contig = (p.ld == p.cols);
  qp.cols = (uint32_t)p.cols;
  qp.g4 = (uint32_t)((p.cols / 16 + 3) / 4);
  qp.seed = p.seed;
  qp.keys = philox_keys(p.seed);
  qp.jbase = p.idx_base >> 2;
  qp.mx_thr = p.mx_thr;
  qp.ts = nullptr;
  qp.ts_copy_out = nullptr;
  qp.codes = reinterpret_cast<uint32_t*>(p.codes);
  qp.scales = p.scales;
  qp.rotated = p.rotated;
  qp.error = s.error;
  qp.deq = p.deq;
  qp.sf_rows = (uint32_t)p.rows;
  qp.sf_groups = (uint32_t)(p.cols / 16);
  qp.g4d = make_fastdiv(qp.g4 > 0u ? qp.g4 : 1u);
  fp.ts_out = ts_out;
  fp.partials = s.partials;
  fp.arrive = s.grid_arrive;
  fp.depart = s.grid_depart;
  fp.error = s.error;
  fp.tiles_per_cta = per;
  const uint64_t ntiles = ((uint64_t)qp.nchunks + 31u) / 32u;
  const uint32_t grid = (uint32_t)((ntiles + per - 1) / per);
  const bool sfmma = p.sf_mma != 0;
  if (p.four_six) {
    if (p.had != 0 || p.deq_mode != 0) return cudaErrorInvalidValue;
    return p.rnd == RND_RTN ? fused_dispatch_sf<RND_RTN, 0, FMT_NV46>(fp, sfmma, grid, smem, st)
                            : fused_dispatch_sf<RND_SR, 0, FMT_NV46>(fp, sfmma, grid, smem, st);
  }
  if (p.deq_mode != 0) {
    if (p.had != 0) return cudaErrorInvalidValue;
    fp.q.deq = p.deq;
#define FP4_FUSED_DQ(R, D) \
    return sfmma ? fused_launch<FMT_NV, R, 0, true, D>(fp, grid, smem, st) : fused_launch<FMT_NV, R, 0, false, D>(fp, grid, smem, st)
    if (p.rnd == RND_RTN) {
      if (p.deq_mode == 1) FP4_FUSED_DQ(RND_RTN, 1);
      FP4_FUSED_DQ(RND_RTN, 2);
    }
    if (p.deq_mode == 1) FP4_FUSED_DQ(RND_SR, 1);
    FP4_FUSED_DQ(RND_SR, 2);
#undef FP4_FUSED_DQ
  }
#define FP4_FUSED_HAD(H)                                                                               \
  return p.rnd == RND_RTN ? fused_dispatch_sf<RND_RTN, H>(fp, sfmma, grid, smem, st)                  \
                          : fused_dispatch_sf<RND_SR, H>(fp, sfmma, grid, smem, st)
  switch (p.had) {
    case 0: FP4_FUSED_HAD(0);
    case 16: FP4_FUSED_HAD(16);
    case 32: FP4_FUSED_HAD(32);
    case 64: FP4_FUSED_HAD(64);
    case 128: FP4_FUSED_HAD(128);
    default: return cudaErrorInvalidValue;
  }
#undef FP4_FUSED_HAD
}

template <int FMT, int RND, bool SFMMA>
static cudaError_t cols_launch(const QColParams& qp, int num_sms, cudaStream_t st) {
  // MXFP4 stochastic rounding: four columns a thread (quantize_cols_mx_sr_kernel)
  constexpr bool kMxSr = FMT == FMT_MX && RND == RND_SR;
  auto kernel = kMxSr ? quantize_cols_mx_sr_kernel<SFMMA> : quantize_cols_kernel<FMT, RND, SFMMA>;
  static int occ = resident_ctas(kernel, 256);
  const uint32_t ntiles = ((qp.R + 127u) / 128u) * ((qp.C + 63u) / 64u);
  uint32_t grid = (uint32_t)num_sms * (uint32_t)occ;
  if (ntiles < grid) grid = ntiles > 0 ? ntiles : 1;
  return launch_kernel(kernel, dim3(grid), dim3(256), 0, st, false, 1u, qp);
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
    qp.nblocks = (uint32_t)(p.rows * (p.cols / bs));
    qp.bpr = make_fastdiv((uint32_t)(p.cols / bs));
    qp.cpr = make_fastdiv((uint32_t)(p.cols / 8));
    qp.ld = p.ld;
    qp.contig = (p.ld == p.cols);
    qp.cols = (uint32_t)p.cols;
    qp.g4 = (uint32_t)((p.cols / bs + 3) / 4);
    qp.seed = p.seed;
    qp.keys = philox_keys(p.seed);
    qp.jbase = p.idx_base >> 2;
    qp.mx_thr = p.mx_thr;
    qp.ts = p.ts;
    qp.ts_copy_out = p.ts_copy_out;
    qp.codes = reinterpret_cast<uint32_t*>(p.codes);
    qp.scales = p.scales;
    qp.rotated = p.rotated;
    qp.error = p.error;
    qp.deq = p.deq;
    qp.sf_rows = (uint32_t)p.rows;
    qp.sf_groups = (uint32_t)(p.cols / bs);
    qp.g4d = make_fastdiv(qp.g4 > 0u ? qp.g4 : 1u);
    if (p.deq_mode != 0) {
      if (p.had != 0 || p.four_six) return cudaErrorInvalidValue;
      if (p.fmt == FMT_MX)
        return p.rnd == RND_RTN ? rows_dispatch_dq<FMT_MX, RND_RTN>(qp, p.deq_mode, sfmma, num_sms, st)
                                : rows_dispatch_dq<FMT_MX, RND_SR>(qp, p.deq_mode, sfmma, num_sms, st);
      return p.rnd == RND_RTN ? rows_dispatch_dq<FMT_NV, RND_RTN>(qp, p.deq_mode, sfmma, num_sms, st)
                              : rows_dispatch_dq<FMT_NV, RND_SR>(qp, p.deq_mode, sfmma, num_sms, st);
    }
    if (p.fmt == FMT_MX)
      return p.rnd == RND_RTN ? rows_dispatch_had<FMT_MX, RND_RTN>(qp, p.had, sfmma, num_sms, st)
                              : rows_dispatch_had<FMT_MX, RND_SR>(qp, p.had, sfmma, num_sms, st);
    if (p.four_six) {
      if (p.had != 0) return cudaErrorInvalidValue;
      return p.rnd == RND_RTN ? rows_dispatch_sf<FMT_NV46, RND_RTN, 0>(qp, sfmma, num_sms, st)
                              : rows_dispatch_sf<FMT_NV46, RND_SR, 0>(qp, sfmma, num_sms, st);
    }
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
  qp.keys = philox_keys(p.seed);
  qp.jbase = p.idx_base >> 2;
  qp.mx_thr = p.mx_thr;
  qp.ts = p.ts;
  qp.ts_copy_out = p.ts_copy_out;
  qp.codes = p.codes;
  qp.scales = p.scales;
  if (p.fmt == FMT_MX)
    return p.rnd == RND_RTN ? cols_dispatch<FMT_MX, RND_RTN>(qp, sfmma, num_sms, st)
                            : cols_dispatch<FMT_MX, RND_SR>(qp, sfmma, num_sms, st);
  if (p.four_six)
    return p.rnd == RND_RTN ? cols_dispatch<FMT_NV46, RND_RTN>(qp, sfmma, num_sms, st)
                            : cols_dispatch<FMT_NV46, RND_SR>(qp, sfmma, num_sms, st);
  return p.rnd == RND_RTN ? cols_dispatch<FMT_NV, RND_RTN>(qp, sfmma, num_sms, st)
                          : cols_dispatch<FMT_NV, RND_SR>(qp, sfmma, num_sms, st);
}

template <int FMT, int RND, bool SFMMA>
static cudaError_t q2d_launch(const Q2Params& qp, int num_sms, cudaStream_t st) {
  auto kernel = quantize_2d_kernel<FMT, RND, SFMMA>;
  static int occ = resident_ctas(kernel, 256);
  constexpr uint32_t TR = FMT == FMT_MX ? 128 : 64;
  const uint64_t tiles = (uint64_t)((qp.R + TR - 1) / TR) * ((qp.C + 63) / 64);
  uint64_t grid = (uint64_t)num_sms * (uint64_t)occ;
  if (tiles < grid) grid = tiles > 0 ? tiles : 1;
  return launch_kernel(kernel, dim3((unsigned)grid), dim3(256), 0, st, false, 1u, qp);
}

template <int FMT>
static cudaError_t q2d_dispatch(const Q2Params& qp, int rnd, bool sfmma, int num_sms, cudaStream_t st) {
  if (rnd == RND_RTN)
    return sfmma ? q2d_launch<FMT, RND_RTN, true>(qp, num_sms, st) : q2d_launch<FMT, RND_RTN, false>(qp, num_sms, st);
  return sfmma ? q2d_launch<FMT, RND_SR, true>(qp, num_sms, st) : q2d_launch<FMT, RND_SR, false>(qp, num_sms, st);
}

cudaError_t launch_quantize_2d(const QuantizeParams& p, uint8_t* codes_t, uint8_t* scales_t, int num_sms,
                               cudaStream_t st) {
  const int bs = p.fmt == FMT_MX ? 32 : 16;
  Q2Params qp;
  qp.x = static_cast<const uint16_t*>(p.x);
  qp.R = (uint32_t)p.rows;
  qp.C = (uint32_t)p.cols;
  qp.ld = p.ld;
  qp.seed = p.seed;
  qp.keys = philox_keys(p.seed);
  qp.mx_thr = p.mx_thr;
  qp.ts = p.ts;
  qp.ts_copy_out = p.ts_copy_out;
  qp.codes = p.codes;
  qp.scales = p.scales;
  qp.codes_t = codes_t;
  qp.scales_t = scales_t;
  qp.g4 = (uint32_t)((p.cols / bs + 3) / 4);
  qp.g4_t = (uint32_t)((p.rows / bs + 3) / 4);
  const bool sfmma = p.sf_mma != 0;
  return p.fmt == FMT_MX ? q2d_dispatch<FMT_MX>(qp, p.rnd, sfmma, num_sms, st)
                         : q2d_dispatch<FMT_NV>(qp, p.rnd, sfmma, num_sms, st);
}

// Direct stores, except for fp32 outputs well beyond L2 (> 96 MB), which stream to HBM faster
// through the staging ring and bulk stores (measured: 8192^2 fp32 53.6 us staged, 58.7 us direct;
// 8192^2 bf16 with tensor-core-layout scales 41.4 us staged, 35.2 us direct).
template <int FMT, bool SFMMA, bool BF16>
static cudaError_t deq_launch(const DeqParams& dp, int num_sms, cudaStream_t st) {
  const bool big_f32 = !BF16 && (uint64_t)dp.nchunks * 32u > 96ull * 1024 * 1024;
  if (!big_f32) {
    auto direct = dequantize_direct_kernel<FMT, SFMMA, BF16>;
    static const int occ_d = resident_ctas(direct, 256);
    const uint32_t want = (dp.nchunks + 256u * kDeqDirectUnroll - 1) / (256u * kDeqDirectUnroll);
    uint32_t grid = (uint32_t)num_sms * (uint32_t)occ_d;
    if (want < grid) grid = want > 0 ? want : 1;
    return launch_kernel(direct, dim3(grid), dim3(256), 0, st, false, 1u, dp);
  }
  auto kernel = dequantize_stream_kernel<FMT, SFMMA, BF16>;
  constexpr int smem = kDeqStages * kDeqTileChunks * (BF16 ? 16 : 32);
  static const int occ = [&] {
    int n = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kDeqThreads, smem) != cudaSuccess || n < 1) n = 1;
    return n;
  }();
  const uint32_t ntiles = (dp.nchunks + kDeqTileChunks - 1) / kDeqTileChunks;
  uint32_t grid = (uint32_t)num_sms * (uint32_t)occ;
  if (ntiles < grid) grid = ntiles > 0 ? ntiles : 1;
  return launch_kernel(kernel, dim3(grid), dim3(kDeqThreads), (size_t)smem, st, false, 1u, dp);
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
