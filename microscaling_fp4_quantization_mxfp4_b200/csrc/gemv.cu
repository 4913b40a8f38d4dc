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
  unsigned* error;       // device error word (bit 0: a shared-memory staging wait expired)
};

// Scale of block g of row r (tensor-core layout) as an fp32 multiplier: the E4M3 value (NV) or
// 2^(e - 127) (MX).
template <int FMT>
__device__ __forceinline__ float block_scale(const uint8_t* sf, uint32_t r, uint32_t g, uint32_t g4) {
  const uint32_t byte = sf[sf_mma_offset(r, g, g4)];
  return FMT == FMT_MX ? mx_scale_value(byte) : e4m3_value(byte);
}

// The activation rows as f16x2 values in shared memory (act: per row, one 16-byte granule of four
// f16x2 values per code word, the four granules of a 32-code chunk c in the order
// q ^ ((c >> 1) & 3), so that the eight lanes of a quarter warp, chunks c .. c + 7 64 bytes apart,
// read distinct bank groups) and their block scales as fp32 multipliers (asc), by all threads.
template <int FMT, int M>
__device__ __forceinline__ void stage_activations(const GemvParams& p, uint4* act, float* asc) {
  constexpr uint32_t BS = FMT == FMT_MX ? 32u : 16u;
  const uint32_t K = p.K, G = K / BS, K8 = K / 8u;
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
}

// Scale byte(s) of chunk c (NVFP4: groups 2c and 2c + 1 as one 16-bit word) of weight row `row` in
// the tensor-core layout; 0 past the row's end.
template <int FMT>
__device__ __forceinline__ uint32_t chunk_scale(const GemvParams& p, uint32_t row, uint32_t c, uint32_t nchunks) {
  if (c >= nchunks) return 0u;
  const uint32_t rb = ((((row >> 7) * p.g4) << 9) + ((row & 31u) << 4) + (((row >> 5) & 3u) << 2));
  if (FMT == FMT_MX) return (uint32_t)__ldg(p.b_sf + rb + ((c >> 2) << 9) + (c & 3u));
  return (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(p.b_sf + rb + ((c >> 1) << 9) + ((c & 1u) << 1)));
}

// acc[m] += the products of one 16-byte chunk c of a weight row (32 codes: one MXFP4 or two NVFP4
// blocks, w its code words, s its scale byte(s) as loaded) with activation row m: exact f16x2 sums
// of eight products, one fp32 rounding per block.
template <int FMT, int M>
__device__ __forceinline__ void chunk_dot(const uint4& w, uint32_t s, uint32_t c, const uint4* act, const float* asc,
                                          uint32_t K8, uint32_t G, uint32_t swz, float (&acc)[M]) {
  const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
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
    const float sb = mx_scale_value(s);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float2 s0 = __half22float2(hs[m][0]), s1 = __half22float2(hs[m][1]);
      const float bsum = __fadd_rn(__fadd_rn(s0.x, s0.y), __fadd_rn(s1.x, s1.y));   // exact
      acc[m] = __fmaf_rn(bsum, __fmul_rn(asc[m * G + c], sb), acc[m]);
    }
  } else {
    uint32_t hsb;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hsb) : "h"((uint16_t)s));
    const float2 sb = __half22float2(*reinterpret_cast<const __half2*>(&hsb));
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float2 s0 = __half22float2(hs[m][0]), s1 = __half22float2(hs[m][1]);
      acc[m] = __fmaf_rn(__fadd_rn(s0.x, s0.y), __fmul_rn(asc[m * G + 2u * c], sb.x), acc[m]);
      acc[m] = __fmaf_rn(__fadd_rn(s1.x, s1.y), __fmul_rn(asc[m * G + 2u * c + 1u], sb.y), acc[m]);
    }
  }
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
#pragma unroll
    for (int u = 0; u < (int)U; ++u) {
      const uint32_t c = c0 + 32u * u;
      w[u] = c < nchunks ? __ldg(brow + c) : make_uint4(0u, 0u, 0u, 0u);
      s[u] = chunk_scale<FMT>(p, row, c, nchunks);
    }
  };
  if (n < p.N) load(n, cb, wc, sc);                     // in flight while the activations are converted
  stage_activations<FMT, M>(p, act, asc);
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
        chunk_dot<FMT, M>(wc[u], sc[u], c, act, asc, K8, G, swz, acc);
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

// ------------------------------------------------- whole-slice staging ----
// For few, long weight rows: gemv_kernel gives each CTA kGemvWarps rows, so N = 1000 rows occupy
// only 63 SMs.  Here every SM gets a CTA and an even share of the rows (whole rows), which the
// bulk-copy engine fetches into shared memory at the start in kGemvPieces copies, each completing
// on its own mbarrier; the warps take the rows n0 + warp, n0 + warp + kGemvWarps, ... from shared
// memory as their pieces land.  Same lane-to-chunk mapping, scale loads and arithmetic as
// gemv_kernel, so the outputs are bit-identical.  Graph-replayed, N = 1000, K = 11008: NVFP4
// 8.85 -> 5.52 us, MXFP4 6.72 -> 5.02 us.  For the Llama-7B decode shapes, where gemv_kernel already
// fills every SM twice over, this kernel measured about 1.3 us slower (NVFP4 11008 x 4096: 11.5
// against 12.8 us): its CTA holds up to 226 KB of shared memory, so the next launch's CTAs cannot
// start on an SM until it has left, while gemv_kernel's small CTAs overlap their set-up with the
// previous launch's tail.
constexpr int kGemvPieces = 8;
constexpr size_t kGemvBulkMaxSmem = 226 * 1024;

template <int FMT, bool BF16>
__global__ void __launch_bounds__(32 * kGemvWarps, 1) gemv_bulk_kernel(GemvParams p) {
  constexpr uint32_t BS = FMT == FMT_MX ? 32u : 16u;
  constexpr uint32_t U = kGemvUnroll;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ __align__(8) uint64_t piece_bar[kGemvPieces];
  const uint32_t K = p.K, G = K / BS, K8 = K / 8u, nchunks = K / 32u, row_bytes = K / 2u;
  uint4* act = reinterpret_cast<uint4*>(smem);                                       // [K/8]
  float* asc = reinterpret_cast<float*>(smem + (size_t)K8 * 16u);                    // [K/BS]
  uint8_t* slice = smem + (size_t)K8 * 16u + (((size_t)G * 4u + 15u) & ~(size_t)15u);  // [rows][K/2]
  const uint32_t n0 = (uint32_t)(((unsigned long long)p.N * blockIdx.x) / gridDim.x);
  const uint32_t n1 = (uint32_t)(((unsigned long long)p.N * (blockIdx.x + 1u)) / gridDim.x);
  const uint32_t rows = n1 - n0, rp = (rows + kGemvPieces - 1u) / kGemvPieces;       // rows a piece
  pdl_trigger();
  if (threadIdx.x == 0) {
    for (int k = 0; k < kGemvPieces; ++k) mbar_init(smem_addr(&piece_bar[k]), 1);
    mbar_init_fence();
  }
  pdl_wait();
  if (threadIdx.x == 0) {
    for (uint32_t k = 0; k < (uint32_t)kGemvPieces; ++k) {
      const uint32_t a = min(rows, k * rp), b = min(rows, (k + 1u) * rp);
      const uint32_t bar = smem_addr(&piece_bar[k]);
      if (b > a) {
        mbar_expect_tx(bar, (b - a) * row_bytes);
        bulk_g2s(smem_addr(slice + (size_t)a * row_bytes), p.b + (size_t)(n0 + a) * row_bytes, (b - a) * row_bytes,
                 bar);
      } else {
        mbar_arrive(bar);                                    // empty piece: complete its phase
      }
    }
  }
  const int lane = threadIdx.x & 31;
  const uint32_t swz = ((uint32_t)lane >> 1) & 3u;      // (c >> 1) & 3 for every chunk c of this lane
  uint32_t n = n0 + (threadIdx.x >> 5), cb = (uint32_t)lane;
  uint32_t sc[U], sn[U];
  if (n < n1) {                                         // in flight while the activations are converted
#pragma unroll
    for (int u = 0; u < (int)U; ++u) sc[u] = chunk_scale<FMT>(p, n, cb + 32u * u, nchunks);
  }
  stage_activations<FMT, 1>(p, act, asc);
  __syncthreads();
  const float alpha = FMT == FMT_MX ? 1.0f : __fmul_rn(*p.a_ts, *p.b_ts);
  float acc[1] = {0.0f};
  uint32_t landed = 0;                                  // pieces this warp has seen complete
  bool ok = true;
  while (n < n1) {
    // next segment: the rest of this row, else the start of the warp's next row
    uint32_t nn = n, nc = cb + 32u * U;
    if (nc >= nchunks) {
      nn = n + kGemvWarps;
      nc = (uint32_t)lane;
    }
    if (nn < n1) {
#pragma unroll
      for (int u = 0; u < (int)U; ++u) sn[u] = chunk_scale<FMT>(p, nn, nc + 32u * u, nchunks);
    }
    for (const uint32_t piece = (n - n0) / rp; landed <= piece; ++landed) {   // warp-uniform
      int w = 1;
      if (lane == 0) w = mbar_wait_bounded(smem_addr(&piece_bar[landed]), 0u) ? 1 : 0;
      if (!__shfl_sync(0xFFFFFFFFu, w, 0)) {
        ok = false;
        break;
      }
    }
    if (!ok) break;
    __syncwarp();
    const uint4* wrow = reinterpret_cast<const uint4*>(slice + (size_t)(n - n0) * row_bytes);
#pragma unroll
    for (int u = 0; u < (int)U; ++u) {
      const uint32_t c = cb + 32u * u;
      if (c < nchunks) chunk_dot<FMT, 1>(wrow[c], sc[u], c, act, asc, K8, G, swz, acc);
    }
    if (nn != n) {                                      // the row is complete: reduce, store, reset
#pragma unroll
      for (int d = 16; d >= 1; d >>= 1) acc[0] = __fadd_rn(acc[0], __shfl_xor_sync(0xFFFFFFFFu, acc[0], d));
      if (lane == 0) {
        const float v = __fmul_rn(acc[0], alpha);
        if (BF16) {
          reinterpret_cast<__nv_bfloat16*>(p.y)[n] = __float2bfloat16_rn(v);
        } else {
          reinterpret_cast<float*>(p.y)[n] = v;
        }
      }
      acc[0] = 0.0f;
    }
    n = nn;
    cb = nc;
#pragma unroll
    for (int u = 0; u < (int)U; ++u) sc[u] = sn[u];
  }
  if (!ok && lane == 0 && p.error != nullptr) atomicOr(p.error, 1u);
  if (threadIdx.x == 0) {                               // every copy lands before the CTA may exit
    for (int k = 0; k < kGemvPieces; ++k) mbar_wait_bounded(smem_addr(&piece_bar[k]), 0u);
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

// Dynamic shared memory of gemv_bulk_kernel: f16 activations, block scales (16-byte rounded) and
// the largest CTA's rows, for a grid of min(SMs, N) CTAs.
size_t gemv_bulk_smem(const GemmParams& p, int num_sms) {
  const int64_t bs = p.fmt == FMT_MX ? 32 : 16;
  const int64_t grid = std::min<int64_t>(num_sms, p.N);
  const int64_t rows = (p.N + grid - 1) / grid;
  return (size_t)(p.K * 2 + ((p.K / bs) * 4 + 15) / 16 * 16 + rows * (p.K / 2));
}

template <int FMT, bool BF16>
cudaError_t gemv_bulk_launch(const GemvParams& gp, size_t smem, int num_sms, cudaStream_t st) {
  auto kernel = gemv_bulk_kernel<FMT, BF16>;
  static const cudaError_t attr =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemvBulkMaxSmem);
  if (attr != cudaSuccess) return attr;
  const uint32_t grid = gp.N < (uint32_t)num_sms ? gp.N : (uint32_t)num_sms;
  return launch_kernel(kernel, dim3(grid), dim3(32 * kGemvWarps), smem, st, false, 1u, gp);
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
  gp.error = p.error;
  // one activation row whose weights would leave more than half of the SMs idle under gemv_kernel,
  // with at least 16 KB of them for each SM that fit its shared memory: stage each CTA's rows whole
  const size_t bsmem = gemv_bulk_smem(p, num_sms);
  const int64_t streaming_ctas = (p.N + kGemvWarps - 1) / kGemvWarps;
  const int64_t slice = (p.N + num_sms - 1) / num_sms * (p.K / 2);
  if (p.M == 1 && 2 * streaming_ctas < num_sms && slice >= 16384 && bsmem <= kGemvBulkMaxSmem &&
      (reinterpret_cast<uintptr_t>(p.b) & 15u) == 0) {
    if (p.fmt == FMT_MX)
      return p.y_bf16 ? gemv_bulk_launch<FMT_MX, true>(gp, bsmem, num_sms, st)
                      : gemv_bulk_launch<FMT_MX, false>(gp, bsmem, num_sms, st);
    return p.y_bf16 ? gemv_bulk_launch<FMT_NV, true>(gp, bsmem, num_sms, st)
                    : gemv_bulk_launch<FMT_NV, false>(gp, bsmem, num_sms, st);
  }
  const size_t smem = gemv_smem(p);
  if (p.fmt == FMT_MX)
    return p.y_bf16 ? gemv_dispatch_m<FMT_MX, true>(gp, smem, num_sms, st)
                    : gemv_dispatch_m<FMT_MX, false>(gp, smem, num_sms, st);
  return p.y_bf16 ? gemv_dispatch_m<FMT_NV, true>(gp, smem, num_sms, st)
                  : gemv_dispatch_m<FMT_NV, false>(gp, smem, num_sms, st);
}

}  // namespace fp4lib
