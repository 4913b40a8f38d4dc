// Block-scaled FP4 GEMM for a single activation row on the CUDA cores (the
// kernel takes any small row count M as a template parameter; launch_gemm
// sends it M = 1): Y[m, n] = alpha * sum_k a[m, k] * b[n, k], the weights b
// streamed from HBM once ("Bridging the Gap Between Promise and Performance for
// Microscaling FP4 Quantization", Abstract: FP4 inference on B200, where
// decoding one token is a weight stream).
//
// At M = 1 a tensor-core tile would be almost all padding and the per-k-tile
// tensor-memory scale copies, not HBM, bound it; here every product is exact.
// E2M1 values times E2M1 values are multiples of 1/4 below 36, so a sum of up
// to eight of them (|sum| <= 288, 1152 quarters < 2^11) is exact in f16: each
// half of an f16x2 fused multiply-add accumulator takes eight products of a
// 16-element block (an MXFP4 block fills two accumulators), the halves are
// added in fp32 (exact), and
// fp32(block sum) * (s_a * s_b) enters the fp32 accumulator with one rounding
// per block (s_a * s_b is exact: two E4M3 values, or a power of two).
//
// Layout: one warp per output column n (a weight row); lane l takes the 16-byte
// chunks c = l, l + 32, ... of that row (32 codes: one MX or two NV blocks), so
// each warp load is 512 contiguous bytes.  The activations are converted once
// per CTA into shared memory as f16x2 values; the weights' codes become f16x2
// values with the hardware E2M1 conversion.  Each lane sums its blocks in
// fp32, a shuffle tree adds the 32 lanes, and lane m stores row m times alpha.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>

#include "fp4_device.cuh"
#include "fp4_internal.h"

namespace fp4lib {
namespace {

using namespace fp4dev;

constexpr int kGemvWarps = 16;                 // weight rows in flight per CTA
constexpr int kGemvUnroll = 4;                 // 16-byte chunks a lane loads before using them

struct GemvParams {
  const uint8_t* a;
  const uint8_t* a_sf;
  const float* a_ts;
  const uint8_t* b;
  const uint8_t* b_sf;
  const float* b_ts;
  uint32_t M, N, K;
  uint32_t g4;           // 4-group columns of the scale layout: ceil(K / block / 4)
  void* y;
  int64_t ldy;
};

// Scale of block g of row r (tensor-core layout) as an fp32 multiplier: the E4M3 value (NV) or
// 2^(e - 127) (MX).
template <int FMT>
__device__ __forceinline__ float block_scale(const uint8_t* sf, uint32_t r, uint32_t g, uint32_t g4) {
  const uint32_t byte = sf[sf_mma_offset(r, g, g4)];
  return FMT == FMT_MX ? mx_scale_value(byte) : e4m3_value(byte);
}

template <int FMT, int M, bool BF16>
__global__ void __launch_bounds__(32 * kGemvWarps, M == 1 ? 2 : 1) gemv_kernel(GemvParams p) {
  constexpr uint32_t BS = FMT == FMT_MX ? 32u : 16u;     // elements per scale block
  constexpr uint32_t U = kGemvUnroll;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t K = p.K, G = K / BS, K8 = K / 8u;
  // act: per activation row, one 16-byte granule (four f16x2 values) per code word, the four
  // granules of a 32-code chunk c in the order q ^ ((c >> 1) & 3), so that the eight lanes of a
  // quarter warp (chunks c .. c + 7, 64 bytes apart) read distinct bank groups
  uint4* act = reinterpret_cast<uint4*>(smem);                         // [M][K/8]
  float* asc = reinterpret_cast<float*>(smem + (size_t)M * K8 * 16u);  // [M][K/BS] block scales
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const uint32_t swz = ((uint32_t)lane >> 1) & 3u;      // (c >> 1) & 3 for every chunk c of this lane
  const uint32_t nchunks = K / 32u;                     // 16-byte chunks of a weight row
  const uint32_t warps = gridDim.x * kGemvWarps;
  // this warp's rows n = n0, n0 + warps, ...; a row in segments of U chunks a lane
  // (chunks cb + 32 u); the next segment's loads are issued before the current one is used
  uint32_t n = blockIdx.x * kGemvWarps + (threadIdx.x >> 5), cb = (uint32_t)lane;
  uint4 wc[U], wn[U];
  uint32_t sc[U], sn[U];
  auto load = [&](uint32_t row, uint32_t c0, uint4 (&w)[U], uint32_t (&s)[U]) {
    const uint4* brow = reinterpret_cast<const uint4*>(p.b + (size_t)row * (K / 2u));
    const uint32_t rb = ((((row >> 7) * p.g4) << 9) + ((row & 31u) << 4) + (((row >> 5) & 3u) << 2));
#pragma unroll
    for (int u = 0; u < (int)U; ++u) {
      const uint32_t c = c0 + 32u * u;
      const bool ok = c < nchunks;
      w[u] = ok ? __ldg(brow + c) : make_uint4(0u, 0u, 0u, 0u);
      if (FMT == FMT_MX) {
        s[u] = ok ? (uint32_t)__ldg(p.b_sf + rb + ((c >> 2) << 9) + (c & 3u)) : 0u;
      } else {                                                       // groups 2c and 2c + 1
        s[u] = ok ? (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(p.b_sf + rb + ((c >> 1) << 9) + ((c & 1u) << 1)))
                  : 0u;
      }
    }
  };
  if (n < p.N) load(n, cb, wc, sc);                     // in flight while the activations are converted
  for (uint32_t i = threadIdx.x; i < M * K8; i += blockDim.x) {
    const uint32_t m = i / K8, k8 = i - m * K8, c = k8 >> 2;
    uint32_t h[4];
    e2m1x8_to_f16x2(reinterpret_cast<const uint32_t*>(p.a + (size_t)m * (K / 2u))[k8], h);
    act[m * K8 + 4u * c + ((k8 & 3u) ^ ((c >> 1) & 3u))] = make_uint4(h[0], h[1], h[2], h[3]);
  }
  for (uint32_t i = threadIdx.x; i < M * G; i += blockDim.x) {
    const uint32_t m = i / G, g = i - m * G;
    asc[i] = block_scale<FMT>(p.a_sf, m, g, p.g4);
  }
  __syncthreads();
  if (n >= p.N) return;
  const float alpha = FMT == FMT_MX ? 1.0f : __fmul_rn(*p.a_ts, *p.b_ts);
  float acc[M];
#pragma unroll
  for (int m = 0; m < M; ++m) acc[m] = 0.0f;
  for (;;) {
    // next segment: the rest of this row, else the start of the warp's next row
    uint32_t nn = n, nc = cb + 32u * U;
    if (nc >= nchunks) {
      nn = n + warps;
      nc = (uint32_t)lane;
    }
    if (nn < p.N) load(nn, nc, wn, sn);
#pragma unroll
    for (int u = 0; u < (int)U; ++u) {
      const uint32_t c = cb + 32u * u;
      if (c < nchunks) {
        const uint32_t w4[4] = {wc[u].x, wc[u].y, wc[u].z, wc[u].w};
        __half2 hs[M][2];                               // exact f16x2 sums: [block or half-block]
#pragma unroll
        for (int m = 0; m < M; ++m) hs[m][0] = hs[m][1] = __float2half2_rn(0.0f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {                   // 8 codes: elements 8q .. 8q + 7 of the chunk
          uint32_t h[4];
          e2m1x8_to_f16x2(w4[q], h);
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const uint4 av = act[m * K8 + 4u * c + ((uint32_t)q ^ swz)];
            const uint32_t a4[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
              hs[m][q >> 1] = __hfma2(*reinterpret_cast<const __half2*>(&h[j]),
                                      *reinterpret_cast<const __half2*>(&a4[j]), hs[m][q >> 1]);
          }
        }
        if (FMT == FMT_MX) {
          const float sb = mx_scale_value(sc[u]);
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float2 s0 = __half22float2(hs[m][0]), s1 = __half22float2(hs[m][1]);
            const float bsum = __fadd_rn(__fadd_rn(s0.x, s0.y), __fadd_rn(s1.x, s1.y));   // exact
            acc[m] = __fmaf_rn(bsum, __fmul_rn(asc[m * G + c], sb), acc[m]);
          }
        } else {
          uint32_t hsb;
          asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hsb) : "h"((uint16_t)sc[u]));
          const float2 sb = __half22float2(*reinterpret_cast<const __half2*>(&hsb));
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float2 s0 = __half22float2(hs[m][0]), s1 = __half22float2(hs[m][1]);
            acc[m] = __fmaf_rn(__fadd_rn(s0.x, s0.y), __fmul_rn(asc[m * G + 2u * c], sb.x), acc[m]);
            acc[m] = __fmaf_rn(__fadd_rn(s1.x, s1.y), __fmul_rn(asc[m * G + 2u * c + 1u], sb.y), acc[m]);
          }
        }
      }
    }
    if (nn != n) {                                      // the row is complete: reduce, store, reset
#pragma unroll
      for (int m = 0; m < M; ++m) {
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) acc[m] = __fadd_rn(acc[m], __shfl_xor_sync(0xFFFFFFFFu, acc[m], d));
      }
      if (lane < M) {
        float v = acc[0];
#pragma unroll
        for (int m = 1; m < M; ++m) v = lane == m ? acc[m] : v;
        v = __fmul_rn(v, alpha);
        if (BF16) {
          reinterpret_cast<__nv_bfloat16*>(p.y)[(size_t)lane * p.ldy + n] = __float2bfloat16_rn(v);
        } else {
          reinterpret_cast<float*>(p.y)[(size_t)lane * p.ldy + n] = v;
        }
      }
#pragma unroll
      for (int m = 0; m < M; ++m) acc[m] = 0.0f;
    }
    if (nn >= p.N) break;
    n = nn;
    cb = nc;
#pragma unroll
    for (int u = 0; u < (int)U; ++u) {
      wc[u] = wn[u];
      sc[u] = sn[u];
    }
  }
}

size_t gemv_smem(const GemmParams& p) {
  const int64_t bs = p.fmt == FMT_MX ? 32 : 16;
  return (size_t)(p.M * p.K * 2 + p.M * (p.K / bs) * 4);   // f16 activations, block scales
}

template <int FMT, int M, bool BF16>
cudaError_t gemv_launch(const GemvParams& gp, size_t smem, int num_sms, cudaStream_t st) {
  auto kernel = gemv_kernel<FMT, M, BF16>;
  static const cudaError_t attr =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemvMaxSmem);
  if (attr != cudaSuccess) return attr;
  // resident CTAs per SM: the launch bounds' 2 (M = 1) or 1, fewer if shared memory runs out
  const size_t fit = (size_t)(227 * 1024) / (smem + 1024);
  const uint32_t per_sm = (uint32_t)std::max<size_t>(1, std::min<size_t>(M == 1 ? 2 : 1, fit));
  const uint32_t need = (gp.N + kGemvWarps - 1) / kGemvWarps;
  const uint32_t cap = (uint32_t)num_sms * per_sm;
  return launch_kernel(kernel, dim3(need < cap ? need : cap), dim3(32 * kGemvWarps), smem, st, false, 1u, gp);
}

template <int FMT, bool BF16>
cudaError_t gemv_dispatch_m(const GemvParams& gp, size_t smem, int num_sms, cudaStream_t st) {
  static_assert(kGemvMaxM == 1, "instantiate the kernel for every row count up to kGemvMaxM");
  return gemv_launch<FMT, 1, BF16>(gp, smem, num_sms, st);
}

}  // namespace

bool gemv_applies(const GemmParams& p) {
  return p.q_out == 0 && p.M >= 1 && p.M <= kGemvMaxM && p.K % 64 == 0 && gemv_smem(p) <= kGemvMaxSmem &&
         ((p.N + 127) / 128) * 128 * (p.K / 16) < ((int64_t)1 << 31);      // 32-bit scale offsets
}

cudaError_t launch_gemv(const GemmParams& p, int num_sms, cudaStream_t st) {
  if (!gemv_applies(p)) return cudaErrorInvalidValue;
  GemvParams gp;
  gp.a = p.a;
  gp.a_sf = p.a_sf;
  gp.a_ts = p.a_ts;
  gp.b = p.b;
  gp.b_sf = p.b_sf;
  gp.b_ts = p.b_ts;
  gp.M = (uint32_t)p.M;
  gp.N = (uint32_t)p.N;
  gp.K = (uint32_t)p.K;
  gp.g4 = (uint32_t)((p.K / (p.fmt == FMT_MX ? 32 : 16) + 3) / 4);
  gp.y = p.y;
  gp.ldy = p.ldy;
  const size_t smem = gemv_smem(p);
  if (p.fmt == FMT_MX)
    return p.y_bf16 ? gemv_dispatch_m<FMT_MX, true>(gp, smem, num_sms, st)
                    : gemv_dispatch_m<FMT_MX, false>(gp, smem, num_sms, st);
  return p.y_bf16 ? gemv_dispatch_m<FMT_NV, true>(gp, smem, num_sms, st)
                  : gemv_dispatch_m<FMT_NV, false>(gp, smem, num_sms, st);
}

}  // namespace fp4lib
