// Block-scaled FP4 x FP4 GEMM with fp32 accumulation on the sm_100a tensor
// cores (tcgen05), fed by TMA.
//
// Method: "Bridging the Gap Between Promise and Performance for Microscaling
// FP4 Quantization", Abstract (FP4 GEMM kernels on B200 for MXFP4/NVFP4);
// "Oscillation-Reduced MXFP4 Training for Vision Transformers", Abstract (MX
// matmuls on Blackwell).  Y[M,N] = alpha * sum_k (cA*sA)(cB*sB), both operands
// K-major ("TN"); the quantizer writes its scale bytes straight into the
// tensor-core scale layout, so nothing is reshuffled here.
//
// Design (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: A/B code tiles (128-byte rows, 128B swizzle) and
//               the scale-factor atoms (plain bulk copies) into a STAGES-deep
//               shared-memory ring guarded by full/empty mbarriers.
//   warp 1      allocates tensor memory; one thread issues 4 block-scaled MMAs
//               (K = 64 each) per 256-wide k-tile, committing to the stage's
//               empty barrier and to the scale buffer's empty barrier.
//   last warp   scale-factor copier: one thread copies each stage's scale
//               atoms to one of four tensor-memory scale buffers
//               (tcgen05.cp 32x128b.warpx4) ahead of the MMAs.  The copies
//               run on their own path, so issuing them from a separate thread
//               lets them overlap the previous k-tiles' MMAs instead of
//               queueing between them (measured: 22-28% faster than copying
//               from the MMA thread).
//   other warps epilogue: tcgen05.ld the fp32 accumulator (two accumulator
//               buffers in tensor memory when BN = 128 so the next tile's MMAs
//               overlap the stores), release it, multiply by alpha and store:
//               bf16 through a 4 KB 128B-swizzled shared-memory box per warp
//               and TMA stores (full-line writes; short-K shapes are bound by
//               the output write), fp32 or unaligned rows with direct stores.
// Every mbarrier wait is bounded; on expiry the CTA raises a shared abort
// flag and a device error word, drains its own copies and MMAs, frees tensor
// memory and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "fp4_device.cuh"
#include "fp4_internal.h"

namespace fp4lib {
namespace {

constexpr int BM = 128;
constexpr int BK = 256;               // fp4 elements per k-tile (128 bytes per row)
constexpr int BK_BYTES = BK / 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCols = 48;      // one scale-factor buffer: SFA (<= 16 cols) then SFB (<= 32 cols)
constexpr uint32_t kSfBufs = 4;       // scale buffers in tensor memory (after the accumulators)
constexpr unsigned long long kWaitLimitNs = 4000000000ull;   // 4 s per wait
constexpr int kSmemRing = 220 * 1024;   // operand stages + output staging, below the 227 KB a CTA can have
constexpr int kEpiStage = 4096;         // one 32-row x 64-column bf16 box, 128B-swizzled

template <int FMT>
struct FmtTraits {
  static constexpr int kBlock = FMT == FMT_MX ? 32 : 16;
  static constexpr int kAtomsPerKTile = BK / kBlock / 4;     // 128x4 scale atoms per 128 rows per k-tile
};

template <int BN, int FMT, bool EPI = true>
struct Cfg {
  static constexpr int kAccStages = BN == 128 ? 2 : 1;
  static constexpr int kEpiWarps = BN == 256 ? 8 : 4;          // each epilogue warp drains 128 columns
  static constexpr int kThreads = 96 + 32 * kEpiWarps;        // producer, MMA, epilogue warps, scale copier
  static constexpr int kSfWarp = 2 + kEpiWarps;
  static constexpr uint32_t kSfBase = (uint32_t)(kAccStages * BN);   // scale buffers after the accumulators
  static_assert(kSfBase + kSfBufs * kSfCols <= kTmemCols, "tensor memory budget");
  static constexpr int kApk = FmtTraits<FMT>::kAtomsPerKTile;
  static constexpr int kABytes = BM * BK_BYTES;
  static constexpr int kBBytes = BN * BK_BYTES;
  static constexpr int kSfaBytes = kApk * 512;
  static constexpr int kSfbBytes = (BN / 128) * kApk * 512;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  // bf16 output staging for TMA stores: 4 KB (32 rows x 128 bytes) per epilogue warp
  static constexpr int kEpiBytes = EPI ? kEpiWarps * kEpiStage : 0;
  static constexpr int kRing = kSmemRing - kEpiBytes;
  static constexpr int kStages = kRing / kStageBytes > 8 ? 8 : kRing / kStageBytes;
  static constexpr int kBarrierBytes = 1024;
  static constexpr int kSmemBytes = 1024 /*alignment slack*/ + kStages * kStageBytes + kEpiBytes + kBarrierBytes;
};

// ------------------------------------------------------------ PTX wrappers --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait: false when the time limit passes or another role raised abort.
// try_wait with a suspend-time hint: the warp sleeps in hardware until the
// phase completes or ~20 us pass, instead of spinning on issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0u;
}
// Critical-path wait (producer, MMA issuer): spin on try_wait, checking the
// abort flag and the time limit every 1024 polls.
__device__ __forceinline__ bool wait_spin(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 0u) {
      if (*abort_flag != 0) return false;
      if (global_timer() - t0 > kWaitLimitNs) return false;
    }
  }
}
// Long waits (epilogue warps): sleep in hardware between polls.
__device__ __noinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort_flag != 0) return false;
    if (global_timer() - t0 > kWaitLimitNs) return false;
  }
}
__device__ __forceinline__ void raise_abort(volatile int* abort_flag, unsigned* error) {
  *abort_flag = 1;
  atomicOr(error, 1u);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

template <int FMT>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
  if (FMT == FMT_MX) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  }
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Waits for this thread's tensor-memory loads into r[4][32].  The registers are in-out operands of
// the wait (and of an empty statement right after it), so the compiler cannot schedule any use of
// them ahead of the wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[4][32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0][0]), "+r"(r[0][1]), "+r"(r[0][2]), "+r"(r[0][3]), "+r"(r[0][4]), "+r"(r[0][5]), "+r"(r[0][6]), "+r"(r[0][7]), "+r"(r[0][8]), "+r"(r[0][9]), "+r"(r[0][10]), "+r"(r[0][11]), "+r"(r[0][12]), "+r"(r[0][13]), "+r"(r[0][14]), "+r"(r[0][15]), "+r"(r[0][16]), "+r"(r[0][17]), "+r"(r[0][18]), "+r"(r[0][19]), "+r"(r[0][20]), "+r"(r[0][21]), "+r"(r[0][22]), "+r"(r[0][23]), "+r"(r[0][24]), "+r"(r[0][25]), "+r"(r[0][26]), "+r"(r[0][27]), "+r"(r[0][28]), "+r"(r[0][29]), "+r"(r[0][30]), "+r"(r[0][31]),
                 "+r"(r[1][0]), "+r"(r[1][1]), "+r"(r[1][2]), "+r"(r[1][3]), "+r"(r[1][4]), "+r"(r[1][5]), "+r"(r[1][6]), "+r"(r[1][7]), "+r"(r[1][8]), "+r"(r[1][9]), "+r"(r[1][10]), "+r"(r[1][11]), "+r"(r[1][12]), "+r"(r[1][13]), "+r"(r[1][14]), "+r"(r[1][15]), "+r"(r[1][16]), "+r"(r[1][17]), "+r"(r[1][18]), "+r"(r[1][19]), "+r"(r[1][20]), "+r"(r[1][21]), "+r"(r[1][22]), "+r"(r[1][23]), "+r"(r[1][24]), "+r"(r[1][25]), "+r"(r[1][26]), "+r"(r[1][27]), "+r"(r[1][28]), "+r"(r[1][29]), "+r"(r[1][30]), "+r"(r[1][31])
               :
               : "memory");
  asm volatile(""
               : "+r"(r[2][0]), "+r"(r[2][1]), "+r"(r[2][2]), "+r"(r[2][3]), "+r"(r[2][4]), "+r"(r[2][5]), "+r"(r[2][6]), "+r"(r[2][7]), "+r"(r[2][8]), "+r"(r[2][9]), "+r"(r[2][10]), "+r"(r[2][11]), "+r"(r[2][12]), "+r"(r[2][13]), "+r"(r[2][14]), "+r"(r[2][15]), "+r"(r[2][16]), "+r"(r[2][17]), "+r"(r[2][18]), "+r"(r[2][19]), "+r"(r[2][20]), "+r"(r[2][21]), "+r"(r[2][22]), "+r"(r[2][23]), "+r"(r[2][24]), "+r"(r[2][25]), "+r"(r[2][26]), "+r"(r[2][27]), "+r"(r[2][28]), "+r"(r[2][29]), "+r"(r[2][30]), "+r"(r[2][31]),
                 "+r"(r[3][0]), "+r"(r[3][1]), "+r"(r[3][2]), "+r"(r[3][3]), "+r"(r[3][4]), "+r"(r[3][5]), "+r"(r[3][6]), "+r"(r[3][7]), "+r"(r[3][8]), "+r"(r[3][9]), "+r"(r[3][10]), "+r"(r[3][11]), "+r"(r[3][12]), "+r"(r[3][13]), "+r"(r[3][14]), "+r"(r[3][15]), "+r"(r[3][16]), "+r"(r[3][17]), "+r"(r[3][18]), "+r"(r[3][19]), "+r"(r[3][20]), "+r"(r[3][21]), "+r"(r[3][22]), "+r"(r[3][23]), "+r"(r[3][24]), "+r"(r[3][25]), "+r"(r[3][26]), "+r"(r[3][27]), "+r"(r[3][28]), "+r"(r[3][29]), "+r"(r[3][30]), "+r"(r[3][31]));
}

// Shared-memory matrix descriptor: K-major operand, 128-byte rows, 128B
// swizzle, 8-row groups 1024 bytes apart (Blackwell descriptor version 1).
// TMA store of one box from shared memory, and bulk-group completion.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One epilogue warp's 32 rows x 128 accumulator columns (r[c][i] = column 32c + i of row
// y0 + lane) -> alpha * value in bf16 -> two 32 x 64 boxes through the warp's 4 KB staging
// buffer (1024-byte aligned, 128B-swizzled: 16-byte chunk j of row i at chunk j ^ (i & 7), the
// layout the tensor map's SWIZZLE_128B expects) -> TMA stores, which clip rows >= M and columns
// >= N.  The buffer is reused for the second box once the first store has read it.
__device__ __forceinline__ void epi_store_bf16_tma(const CUtensorMap* tmap_y, uint8_t* stg, const uint32_t (&r)[4][32],
                                                   float alpha, int x0, int y0, int M, int N, int lane) {
  const uint32_t base = smem_u32(stg) + (uint32_t)lane * 128u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (lane == 0) bulk_wait_read0();        // the previous box's store has read the buffer
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = __fmul_rn(__uint_as_float(r[2 * h + (j >> 2)][(j & 3) * 8 + 2 * i]), alpha);
        const float hi = __fmul_rn(__uint_as_float(r[2 * h + (j >> 2)][(j & 3) * 8 + 2 * i + 1]), alpha);
        w[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
               ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
      }
      const uint32_t dst = base + (uint32_t)(((j ^ (lane & 7)) & 7) * 16);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                   : "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> async-proxy reads
    __syncwarp();
    if (lane == 0 && x0 + 64 * h < N && y0 < M) {       // boxes wholly past the edge are skipped
      tma_store_2d(tmap_y, smem_u32(stg), x0 + 64 * h, y0);
      bulk_commit_group();
    }
  }
}

__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(1024u >> 4) << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// Descriptor of one 512-byte scale atom: 32 rows of 16 bytes, no swizzle,
// 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)(128u >> 4) << 32) |
         ((uint64_t)1u << 46);
}

// Instruction descriptor of the block-scaled MMA: E2M1 x E2M1, K-major
// operands, M = 128, N = BN, scale format UE8M0 (MX) or UE4M3 (NV).
template <int BN, int FMT>
__device__ __forceinline__ uint32_t idesc_base() {
  return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((FMT == FMT_MX ? 1u : 0u) << 23) |
         ((uint32_t)(BM >> 4) << 24);
}

struct KernelArgs {
  const uint8_t* a_sf;
  const uint8_t* b_sf;
  const float* a_ts;
  const float* b_ts;
  void* y;
  int64_t ldy;
  int M, N, K;
  int num_m, num_n;
  int g4;                 // padded k-groups / 4 of both scale tensors
  int vec_store;          // output rows 16-byte aligned: 128-bit stores (2: 32-byte aligned, 256-bit stores)
  int tma_store;          // bf16 output through shared memory and TMA stores (tensor map valid)
  unsigned* error;
  // fused quantization of Y along its rows (kernels with QO != 0): codes [M, N/2], scale bytes in
  // the row-major or tensor-core layout, NVFP4 tensor scale (QO = 2), rounding, MX clip threshold
  uint8_t* q_codes;
  uint8_t* q_scales;
  const float* q_ts;
  int q_sf_mma, q_g4, q_rnd;
  uint32_t q_mx_thr;
  fp4dev::PhiloxKeys q_keys;
};

// One 32-byte store (a whole L2 sector) of eight 32-bit words; dst 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* dst, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Byte offset of the scale of (row m, group g) of the quantized Y.
__device__ __forceinline__ long long q_sf_offset(const KernelArgs& p, int m, int g, int groups) {
  return p.q_sf_mma ? fp4dev::sf_mma_offset(m, g, p.q_g4) : (long long)m * groups + g;
}

// Eight codes of scaled values v[0..7] with RTN or SR (Philox word of element idx0 + i, idx0 % 8 == 0).
__device__ __forceinline__ uint32_t q_codes8(const KernelArgs& p, const float* v, unsigned long long idx0) {
  if (!p.q_rnd) return fp4dev::e2m1x4_rn(v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
  const unsigned long long j = idx0 >> 2;
  const fp4dev::u32x4 a = fp4dev::philox4x32_10((uint32_t)j, (uint32_t)(j >> 32), p.q_keys);
  const fp4dev::u32x4 b = fp4dev::philox4x32_10((uint32_t)(j + 1), (uint32_t)((j + 1) >> 32), p.q_keys);
  const uint32_t n[8] = {fp4dev::e2m1_sr(v[0], a.x), fp4dev::e2m1_sr(v[1], a.y), fp4dev::e2m1_sr(v[2], a.z),
                         fp4dev::e2m1_sr(v[3], a.w), fp4dev::e2m1_sr(v[4], b.x), fp4dev::e2m1_sr(v[5], b.y),
                         fp4dev::e2m1_sr(v[6], b.z), fp4dev::e2m1_sr(v[7], b.w)};
  return fp4dev::pack8_nibbles(n);
}

// Fused output quantization of one thread's 32 accumulator columns n0 .. n0+31 of row m
// (rc: fp32 bit patterns, overwritten): y = alpha * acc is the value the fp32 output would hold;
// blocks run along the row (the next GEMM's contraction axis) with the quantizers' arithmetic --
// QO = 1: one MXFP4 block of 32 (E8M0 exponent with clip threshold q_mx_thr); QO = 2: two NVFP4
// blocks of 16 under the given tensor scale st (y_st = RN(1/st), st_ok = recip_usable(st)).
template <int QO>
__device__ __forceinline__ void epi_quantize32(const KernelArgs& p, uint32_t (&rc)[32], float alpha, float st,
                                               float y_st, bool st_ok, int m, int n0) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(__uint_as_float(rc[i]), alpha);
  const unsigned long long idx0 = (unsigned long long)m * (unsigned)p.N + (unsigned)n0;
  uint32_t w[4];
  if (QO == 1) {
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[i]));
    const uint32_t byte = fp4dev::mx_scale_byte_clip(am, p.q_mx_thr);
    const float inv = fp4dev::mx_inv_scale(byte);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(v[i], inv);           // exact power-of-two scaling
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = am == 0.0f ? 0u : q_codes8(p, v + 8 * k, idx0 + 8 * k);
    p.q_scales[q_sf_offset(p, m, n0 / 32, p.N / 32)] = (uint8_t)byte;
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float x[16];
      float am = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        x[i] = v[16 * h + i];
        am = fmaxf(am, fabsf(x[i]));
      }
      const uint32_t byte = fp4dev::e4m3_rn_sat(fp4dev::nv_scale_arg(am, st, y_st, st_ok));
      const float S = byte == 0u ? 1.0f : __fmul_rn(fp4dev::e4m3_value(byte), st);
      const float2 sy = make_float2(S, fp4dev::recip_usable(S) ? __frcp_rn(S) : 0.0f);
      if (p.q_rnd) fp4dev::nv_divide_block<1, 16>(x, am, sy, x);
      else fp4dev::nv_divide_block<0, 16>(x, am, sy, x);
#pragma unroll
      for (int k = 0; k < 2; ++k) w[2 * h + k] = byte == 0u ? 0u : q_codes8(p, x + 8 * k, idx0 + 16 * h + 8 * k);
      p.q_scales[q_sf_offset(p, m, n0 / 16 + h, p.N / 16)] = (uint8_t)byte;
    }
  }
  *reinterpret_cast<uint4*>(p.q_codes + (size_t)m * (unsigned)(p.N / 2) + n0 / 2) = make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& mt, int& nt) {
  constexpr int kGroup = 8;
  const int band = t / (kGroup * num_n);
  const int first = band * kGroup;
  const int gsize = min(kGroup, num_m - first);
  const int local = t - band * kGroup * num_n;
  mt = first + local % gsize;
  nt = local / gsize;
}

template <int BN, int FMT, bool BF16, int QO = 0>
__global__ void __launch_bounds__(Cfg<BN, FMT>::kThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_y, KernelArgs p) {
  pdl_trigger();
  using C = Cfg<BN, FMT>;
  constexpr int S = C::kStages;
  constexpr int APK = C::kApk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * C::kABytes;
  uint8_t* sSFA = sB + S * C::kBBytes;
  uint8_t* sSFB = sSFA + S * C::kSfaBytes;
  uint8_t* sEpi = sSFB + S * C::kSfbBytes;                       // 1024-byte aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + C::kEpiBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* drain = bars + 2 * S + 4;
  uint64_t* sfdrain = bars + 2 * S + 5;
  uint64_t* sf_full = bars + 2 * S + 6;                 // scale buffer b written (copies landed)
  uint64_t* sf_empty = sf_full + kSfBufs;               // scale buffer b free (its MMAs done)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + kSfBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), C::kEpiWarps);
    }
    mbar_init(smem_u32(drain), 1);
    mbar_init(smem_u32(sfdrain), 1);
    for (uint32_t b = 0; b < kSfBufs; ++b) {
      mbar_init(smem_u32(&sf_full[b]), 1);
      mbar_init(smem_u32(&sf_empty[b]), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();                               // the previous kernel's outputs (our operands) are complete

  const int num_tiles = p.num_m * p.num_n;
  const int nkb = (p.K + BK - 1) / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;   // per-stage bits: ever issued / parity of the last issue
      const int rb_total = (p.N + 127) / 128;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, p.num_m, p.num_n, mt, nt);
        const int rb_here = min(BN / 128, rb_total - nt * (BN / 128));
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_spin(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
            raise_abort(abort_flag, p.error);
            ok = false;
            break;
          }
          const int kvalid = min(BK, p.K - kb * BK);
          const int atoms = (kvalid / FmtTraits<FMT>::kBlock + 3) / 4;
          const uint32_t fb = smem_u32(&full[stage]);
          mbar_expect_tx(fb, (uint32_t)(C::kABytes + C::kBBytes + atoms * 512 * (1 + rb_here)));
          tma_load_2d(smem_u32(sA + stage * C::kABytes), &tmap_a, kb * BK_BYTES, mt * BM, fb);
          tma_load_2d(smem_u32(sB + stage * C::kBBytes), &tmap_b, kb * BK_BYTES, nt * BN, fb);
          bulk_load(smem_u32(sSFA + stage * C::kSfaBytes),
                    p.a_sf + ((size_t)mt * p.g4 + (size_t)kb * APK) * 512, (uint32_t)atoms * 512u, fb);
          for (int rb = 0; rb < rb_here; ++rb)
            bulk_load(smem_u32(sSFB + stage * C::kSfbBytes + rb * APK * 512),
                      p.b_sf + ((size_t)(nt * (BN / 128) + rb) * p.g4 + (size_t)kb * APK) * 512,
                      (uint32_t)atoms * 512u, fb);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // let every copy already issued land before the CTA can exit
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) {
            volatile int never = 0;
            wait_bounded(smem_u32(&full[s]), (issued_parity >> s) & 1u, &never);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      uint32_t ktile_count = 0;   // k-tiles issued so far: picks the scale buffer
      bool ok = true;
      bool any_mma = false;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
        int mt, nt;
        tile_coords(t, p.num_m, p.num_n, mt, nt);
        (void)mt;
        const int acc = local % C::kAccStages;
        const uint32_t use = (uint32_t)(local / C::kAccStages);
        if (!wait_spin(smem_u32(&tempty[acc]), (use & 1u) ^ 1u, abort_flag)) {
          raise_abort(abort_flag, p.error);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          const uint32_t b = ktile_count % kSfBufs, use_b = ktile_count / kSfBufs;
          ++ktile_count;
          // the scale buffer's copies landed (the copier waited for this stage first)
          if (!wait_spin(smem_u32(&sf_full[b]), use_b & 1u, abort_flag) ||
              !wait_spin(smem_u32(&full[stage]), phase, abort_flag)) {
            raise_abort(abort_flag, p.error);
            ok = false;
            break;
          }
          tc_fence_after();
          const int kvalid = min(BK, p.K - kb * BK);
          const uint32_t sfa_col = C::kSfBase + b * kSfCols;
          const uint32_t sfb_col = sfa_col + 16u;
          const uint64_t adesc = desc_sw128(smem_u32(sA + stage * C::kABytes));
          const uint64_t bdesc = desc_sw128(smem_u32(sB + stage * C::kBBytes));
          const int nmma = kvalid / 64;
          for (int j = 0; j < nmma; ++j) {
            uint32_t chunk, sf_id;
            if (FMT == FMT_MX) {      // 2 scales per row per MMA: k-groups 2j, 2j+1
              chunk = (uint32_t)(j >> 1);
              sf_id = (uint32_t)((j & 1) * 2);
            } else {                  // 4 scales per row per MMA
              chunk = (uint32_t)j;
              sf_id = 0u;
            }
            const uint32_t idesc = idesc_base<BN, FMT>() | (sf_id << 29) | (sf_id << 4);
            tc_mma<FMT>(d_tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc,
                        tmem + sfa_col + 4u * chunk, tmem + sfb_col + 4u * chunk * (BN / 128),
                        (kb > 0 || j > 0) ? 1u : 0u);
            any_mma = true;
          }
          tc_commit(smem_u32(&empty[stage]));
          tc_commit(smem_u32(&sf_empty[b]));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(smem_u32(&tfull[acc]));
      }
      if (!ok && any_mma) {
        // wait for the MMAs already issued before tensor memory is released
        tc_commit(smem_u32(drain));
        volatile int never = 0;
        wait_bounded(smem_u32(drain), 0u, &never);
      }
    }
    __syncwarp();
  } else if (warp == C::kSfWarp) {
    // ------------------------------------------------------ scale copier --
    // k-tile n's scale atoms go to buffer n % kSfBufs once the stage has landed and the MMAs
    // that last read that buffer have completed; the commit tells the MMA issuer.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, kt = 0;
      bool ok = true, any_cp = false;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        for (int kb = 0; kb < nkb; ++kb) {
          const uint32_t b = kt % kSfBufs, use_b = kt / kSfBufs;
          ++kt;
          if (!wait_spin(smem_u32(&full[stage]), phase, abort_flag) ||
              !wait_spin(smem_u32(&sf_empty[b]), (use_b & 1u) ^ 1u, abort_flag)) {
            raise_abort(abort_flag, p.error);
            ok = false;
            break;
          }
          tc_fence_after();
          const int kvalid = min(BK, p.K - kb * BK);
          const int atoms = (kvalid / FmtTraits<FMT>::kBlock + 3) / 4;
          const uint32_t sfa_col = C::kSfBase + b * kSfCols;
          const uint32_t sfb_col = sfa_col + 16u;
          for (int i = 0; i < atoms; ++i) {
            tc_cp_sf(tmem + sfa_col + 4u * i, desc_sf(smem_u32(sSFA + stage * C::kSfaBytes + i * 512)));
            for (int rb = 0; rb < BN / 128; ++rb)
              tc_cp_sf(tmem + sfb_col + 4u * (i * (BN / 128) + rb),
                       desc_sf(smem_u32(sSFB + stage * C::kSfbBytes + (rb * APK + i) * 512)));
          }
          tc_commit(smem_u32(&sf_full[b]));
          any_cp = true;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && any_cp) {
        // copies already issued complete before tensor memory is released
        tc_commit(smem_u32(sfdrain));
        volatile int never = 0;
        wait_bounded(smem_u32(sfdrain), 0u, &never);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue --
    // Warp w reads tensor-memory lanes 32*(w%4) .. +31 (its hardware quadrant) and
    // 128 accumulator columns; all 128 values per thread are loaded before the
    // accumulator is released, so the next tile's MMAs start while stores drain.
    const int q = warp & 3;
    const int col0 = ((warp - 2) / 4) * 128;
    const int row_in_tile = q * 32 + lane;
    const float alpha = FMT == FMT_NV ? __fmul_rn(*p.a_ts, *p.b_ts) : 1.0f;
    const float q_st = QO == 2 ? *p.q_ts : 1.0f;
    const float q_yst = __frcp_rn(q_st);
    const bool q_stok = fp4dev::recip_usable(q_st);
    int local = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
      int mt, nt;
      tile_coords(t, p.num_m, p.num_n, mt, nt);
      const int acc = local % C::kAccStages;
      const uint32_t use = (uint32_t)(local / C::kAccStages);
      int ok = 1;
      if (lane == 0) ok = wait_bounded(smem_u32(&tfull[acc]), use & 1u, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) {
        if (lane == 0) raise_abort(abort_flag, p.error);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + col0);
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tbase + (uint32_t)(32 * c), r[c]);
      tmem_ld_wait(r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
      if (QO != 0) {
        const int m = mt * BM + row_in_tile;
        if (m < p.M) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int n0 = nt * BN + col0 + 32 * c;
            if (n0 >= p.N) break;
            epi_quantize32<QO>(p, r[c], alpha, q_st, q_yst, q_stok, m, n0);
          }
        }
        continue;
      }
      if (BF16 && p.tma_store) {
        epi_store_bf16_tma(&tmap_y, sEpi + (warp - 2) * kEpiStage, r, alpha, nt * BN + col0, mt * BM + q * 32, p.M,
                           p.N, lane);
        continue;
      }
      const int m = mt * BM + row_in_tile;
      if (m < p.M) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int n0 = nt * BN + col0 + 32 * c;
          if (n0 >= p.N) break;
          if (BF16) {
            __nv_bfloat16* yr = reinterpret_cast<__nv_bfloat16*>(p.y) + (size_t)m * p.ldy + n0;
            if (p.vec_store == 2 && n0 + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 2; ++v) {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float lo = __fmul_rn(__uint_as_float(r[c][16 * v + 2 * i]), alpha);
                  const float hi = __fmul_rn(__uint_as_float(r[c][16 * v + 2 * i + 1]), alpha);
                  w[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                }
                st_global_v8(yr + 16 * v, w);
              }
            } else if (p.vec_store && n0 + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float lo = __fmul_rn(__uint_as_float(r[c][8 * v + 2 * i]), alpha);
                  const float hi = __fmul_rn(__uint_as_float(r[c][8 * v + 2 * i + 1]), alpha);
                  w[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                }
                reinterpret_cast<uint4*>(yr)[v] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (n0 + i < p.N) yr[i] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(r[c][i]), alpha));
            }
          } else {
            float* yr = reinterpret_cast<float*>(p.y) + (size_t)m * p.ldy + n0;
            if (p.vec_store == 2 && n0 + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(__fmul_rn(__uint_as_float(r[c][8 * v + i]), alpha));
                st_global_v8(yr + 8 * v, w);
              }
            } else if (p.vec_store && n0 + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 8; ++v)
                reinterpret_cast<float4*>(yr)[v] = make_float4(
                    __fmul_rn(__uint_as_float(r[c][4 * v]), alpha), __fmul_rn(__uint_as_float(r[c][4 * v + 1]), alpha),
                    __fmul_rn(__uint_as_float(r[c][4 * v + 2]), alpha), __fmul_rn(__uint_as_float(r[c][4 * v + 3]), alpha));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (n0 + i < p.N) yr[i] = __fmul_rn(__uint_as_float(r[c][i]), alpha);
            }
          }
        }
      }
    }
    if (BF16 && p.tma_store && lane == 0) bulk_wait_all0();     // stores done before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// =========================================== SM-pair (cta_group::2) kernel ===
// A cluster of two CTAs on neighbouring SMs computes a 256 x 256 output tile
// with M = 256 MMAs issued by the even ("leader") CTA.  Each CTA stages its own
// 128 rows of A and 128 of B's 256 rows (the MMA reads A and B from both CTAs'
// shared memory at the same offsets), the scale factors of its A rows, and the
// scale factors of all 256 B rows (each CTA's tensor memory holds its 128 x 256
// accumulator).  Operand bytes per SM per MMA are half those of the 128 x 256
// single-SM tile, and one MMA instruction does twice the work.
//   - Both CTAs' TMA loads signal the leader's full barrier (cta_group::2 form);
//     only the leader's producer posts the expected byte count of the pair.
//   - The leader's MMA commits multicast to both CTAs' empty / accumulator-full
//     barriers; both CTAs' epilogue warps arrive on the leader's
//     accumulator-empty barrier (the follower remotely).
//   - Every role falls through to one cluster barrier before tensor memory is
//     freed, and every wait is bounded.
// No load uses TMA multicast.
namespace pair {

// BN = 256: 256 x 256 cluster tiles, one 256-column accumulator, 8 epilogue
// warps.  BN = 128: 256 x 128 tiles, two 128-column accumulators so the next
// tile's MMAs overlap the epilogue (better when K is short), 4 epilogue warps.
template <int BN, int FMT>
struct Cfg2 {
  static constexpr int kApk = FmtTraits<FMT>::kAtomsPerKTile;
  static constexpr int kAccStages = BN == 128 ? 2 : 1;
  static constexpr int kEpiWarps = BN == 256 ? 8 : 4;
  static constexpr int kThreads = 96 + 32 * kEpiWarps;  // producer, MMA, epilogue warps, scale copier
  static constexpr int kSfWarp = 2 + kEpiWarps;
  static constexpr int kBRows = BN / 2;                  // B rows staged by each CTA
  static constexpr int kSfbBlocks = BN / 128;            // 128-row scale blocks of B per tile
  static constexpr int kABytes = 128 * BK_BYTES;
  static constexpr int kBBytes = kBRows * BK_BYTES;
  static constexpr int kSfaBytes = kApk * 512;
  static constexpr int kSfbBytes = kSfbBlocks * kApk * 512;
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  // No output staging: with K >= 2048 the direct stores hide behind the next tile's MMAs, and the
  // 32 KB a TMA-store staging buffer takes would cost a stage (measured 2-3 % slower).
  static constexpr int kStages = kSmemRing / kStageBytes > 8 ? 8 : kSmemRing / kStageBytes;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 1024;
  static constexpr uint32_t kSfBase = (uint32_t)(kAccStages * BN);   // scale buffers after the accumulators
  static_assert(kSfBase + kSfBufs * kSfCols <= kTmemCols, "tensor memory budget");
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
  return d;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}
// commit of the pair's tensor-core work to a barrier of this CTA only
__device__ __forceinline__ void tc_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
template <int FMT>
__device__ __forceinline__ void tc_mma_pair(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t accumulate) {
  if (FMT == FMT_MX) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  }
}

template <int BN, int FMT, bool BF16, int QO = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg2<BN, FMT>::kThreads, 1)
    fp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                         const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                         KernelArgs p) {
  pdl_trigger();
  using C = Cfg2<BN, FMT>;
  constexpr int S = C::kStages;
  constexpr int APK = C::kApk;
  constexpr int kEpiWarps = C::kEpiWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * C::kABytes;
  uint8_t* sSFA = sB + S * C::kBBytes;
  uint8_t* sSFB = sSFA + S * C::kSfaBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + S * C::kSfbBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* tempty = bars + 2 * S + 2;
  uint64_t* drain = bars + 2 * S + 4;
  uint64_t* sfdrain = bars + 2 * S + 5;
  uint64_t* sf_full = bars + 2 * S + 6;                 // scale buffer b written (copies landed)
  uint64_t* sf_empty = sf_full + kSfBufs;               // scale buffer b free (its MMAs done)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + kSfBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), 2 * kEpiWarps);
    }
    mbar_init(smem_u32(drain), 1);
    mbar_init(smem_u32(sfdrain), 1);
    for (uint32_t b = 0; b < kSfBufs; ++b) {
      mbar_init(smem_u32(&sf_full[b]), 1);
      mbar_init(smem_u32(&sf_empty[b]), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();                  // barriers of both CTAs initialised before any remote signal
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();                          // the previous kernel's outputs (our operands) are complete

  const int num_tiles = p.num_m * p.num_n;            // 256 x BN tiles
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int nkb = p.K / BK;                           // K % 256 == 0 on this path

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = cluster; t < num_tiles && ok; t += nclusters) {
        int mt, nt;
        tile_coords(t, p.num_m, p.num_n, mt, nt);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!wait_spin(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
            raise_abort(abort_flag, p.error);
            ok = false;
            break;
          }
          const uint32_t fb = map_rank(smem_u32(&full[stage]), 0);
          if (leader) mbar_expect_tx(smem_u32(&full[stage]), 2u * (uint32_t)C::kStageBytes);
          tma_load_2d_pair(smem_u32(sA + stage * C::kABytes), &tmap_a, kb * BK_BYTES, mt * 256 + (int)rank * 128, fb);
          tma_load_2d_pair(smem_u32(sB + stage * C::kBBytes), &tmap_b, kb * BK_BYTES,
                           nt * BN + (int)rank * C::kBRows, fb);
          tma_load_2d_pair(smem_u32(sSFA + stage * C::kSfaBytes), &tmap_sfa, 0,
                           (mt * 2 + (int)rank) * p.g4 + kb * APK, fb);
#pragma unroll
          for (int rb = 0; rb < C::kSfbBlocks; ++rb)
            tma_load_2d_pair(smem_u32(sSFB + stage * C::kSfbBytes + rb * APK * 512), &tmap_sfb, 0,
                             (nt * C::kSfbBlocks + rb) * p.g4 + kb * APK, fb);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (leader) --
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      uint32_t ktile_count = 0;
      bool ok = true, any_mma = false;
      for (int t = cluster; t < num_tiles && ok; t += nclusters, ++local) {
        const int acc = local % C::kAccStages;
        const uint32_t use = (uint32_t)(local / C::kAccStages);
        if (!wait_spin(smem_u32(&tempty[acc]), (use & 1u) ^ 1u, abort_flag)) {
          raise_abort(abort_flag, p.error);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          const uint32_t b = ktile_count % kSfBufs, use_b = ktile_count / kSfBufs;
          ++ktile_count;
          if (!wait_spin(smem_u32(&sf_full[b]), use_b & 1u, abort_flag) ||
              !wait_spin(smem_u32(&full[stage]), phase, abort_flag)) {
            raise_abort(abort_flag, p.error);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_col = C::kSfBase + b * kSfCols;
          const uint32_t sfb_col = sfa_col + 16u;
          const uint64_t adesc = desc_sw128(smem_u32(sA + stage * C::kABytes));
          const uint64_t bdesc = desc_sw128(smem_u32(sB + stage * C::kBBytes));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t chunk = FMT == FMT_MX ? (uint32_t)(j >> 1) : (uint32_t)j;
            const uint32_t sf_id = FMT == FMT_MX ? (uint32_t)((j & 1) * 2) : 0u;
            const uint32_t idesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                   ((FMT == FMT_MX ? 1u : 0u) << 23) | ((uint32_t)(256 >> 4) << 24) | (sf_id << 29) |
                                   (sf_id << 4);
            tc_mma_pair<FMT>(d_tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc,
                             tmem + sfa_col + 4u * chunk, tmem + sfb_col + 4u * C::kSfbBlocks * chunk,
                             (kb > 0 || j > 0) ? 1u : 0u);
            any_mma = true;
          }
          tc_commit_pair(smem_u32(&empty[stage]));
          tc_commit_pair_local(smem_u32(&sf_empty[b]));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(smem_u32(&tfull[acc]));
      }
      if (!ok && any_mma) {
        tc_commit_pair(smem_u32(drain));
        volatile int never = 0;
        wait_bounded(smem_u32(drain), 0u, &never);
      }
    }
    __syncwarp();
  } else if (warp == C::kSfWarp) {
    // ------------------------------------------------ scale copier (leader) --
    // The leader's cta_group::2 copies fill the same scale buffer in both CTAs' tensor memory,
    // each from its own shared memory.
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0, kt = 0;
      bool ok = true, any_cp = false;
      for (int t = cluster; t < num_tiles && ok; t += nclusters) {
        for (int kb = 0; kb < nkb; ++kb) {
          const uint32_t b = kt % kSfBufs, use_b = kt / kSfBufs;
          ++kt;
          if (!wait_spin(smem_u32(&full[stage]), phase, abort_flag) ||
              !wait_spin(smem_u32(&sf_empty[b]), (use_b & 1u) ^ 1u, abort_flag)) {
            raise_abort(abort_flag, p.error);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_col = C::kSfBase + b * kSfCols;
          const uint32_t sfb_col = sfa_col + 16u;
#pragma unroll
          for (int i = 0; i < APK; ++i) {
            tc_cp_sf_pair(tmem + sfa_col + 4u * i, desc_sf(smem_u32(sSFA + stage * C::kSfaBytes + i * 512)));
#pragma unroll
            for (int rb = 0; rb < C::kSfbBlocks; ++rb)
              tc_cp_sf_pair(tmem + sfb_col + 4u * (i * C::kSfbBlocks + rb),
                            desc_sf(smem_u32(sSFB + stage * C::kSfbBytes + (rb * APK + i) * 512)));
          }
          tc_commit_pair_local(smem_u32(&sf_full[b]));
          any_cp = true;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && any_cp) {
        tc_commit_pair_local(smem_u32(sfdrain));
        volatile int never = 0;
        wait_bounded(smem_u32(sfdrain), 0u, &never);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue --
    const int q = warp & 3;
    const int col0 = ((warp - 2) / 4) * 128;
    const int row_in_tile = (int)rank * 128 + q * 32 + lane;
    const float alpha = FMT == FMT_NV ? __fmul_rn(*p.a_ts, *p.b_ts) : 1.0f;
    const float q_st = QO == 2 ? *p.q_ts : 1.0f;
    const float q_yst = __frcp_rn(q_st);
    const bool q_stok = fp4dev::recip_usable(q_st);
    int local = 0;
    for (int t = cluster; t < num_tiles; t += nclusters, ++local) {
      int mt, nt;
      tile_coords(t, p.num_m, p.num_n, mt, nt);
      const int acc = local % C::kAccStages;
      const uint32_t use = (uint32_t)(local / C::kAccStages);
      const uint32_t tempty_leader = map_rank(smem_u32(&tempty[acc]), 0);
      int ok = 1;
      if (lane == 0) ok = wait_bounded(smem_u32(&tfull[acc]), use & 1u, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) {
        if (lane == 0) raise_abort(abort_flag, p.error);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + col0);
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tbase + (uint32_t)(32 * c), r[c]);
      tmem_ld_wait(r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader);
      const int m = mt * 256 + row_in_tile;
      if (QO != 0) {
        if (m < p.M) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int n0 = nt * BN + col0 + 32 * c;
            if (n0 >= p.N) break;
            epi_quantize32<QO>(p, r[c], alpha, q_st, q_yst, q_stok, m, n0);
          }
        }
        continue;
      }
      if (m < p.M) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int n0 = nt * BN + col0 + 32 * c;
          if (n0 >= p.N) break;
          if (BF16) {
            __nv_bfloat16* yr = reinterpret_cast<__nv_bfloat16*>(p.y) + (size_t)m * p.ldy + n0;
            if (p.vec_store == 2 && n0 + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 2; ++v) {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float lo = __fmul_rn(__uint_as_float(r[c][16 * v + 2 * i]), alpha);
                  const float hi = __fmul_rn(__uint_as_float(r[c][16 * v + 2 * i + 1]), alpha);
                  w[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                }
                st_global_v8(yr + 16 * v, w);
              }
            } else if (p.vec_store && n0 + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const float lo = __fmul_rn(__uint_as_float(r[c][8 * v + 2 * i]), alpha);
                  const float hi = __fmul_rn(__uint_as_float(r[c][8 * v + 2 * i + 1]), alpha);
                  w[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
                }
                reinterpret_cast<uint4*>(yr)[v] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (n0 + i < p.N) yr[i] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(r[c][i]), alpha));
            }
          } else {
            float* yr = reinterpret_cast<float*>(p.y) + (size_t)m * p.ldy + n0;
            if (p.vec_store == 2 && n0 + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(__fmul_rn(__uint_as_float(r[c][8 * v + i]), alpha));
                st_global_v8(yr + 8 * v, w);
              }
            } else if (p.vec_store && n0 + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 8; ++v)
                reinterpret_cast<float4*>(yr)[v] = make_float4(
                    __fmul_rn(__uint_as_float(r[c][4 * v]), alpha), __fmul_rn(__uint_as_float(r[c][4 * v + 1]), alpha),
                    __fmul_rn(__uint_as_float(r[c][4 * v + 2]), alpha), __fmul_rn(__uint_as_float(r[c][4 * v + 3]), alpha));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (n0 + i < p.N) yr[i] = __fmul_rn(__uint_as_float(r[c][i]), alpha);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();                  // neither CTA frees tensor memory or exits while the pair is busy
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace pair

// ================================== split-K clusters (too few output tiles) ===
// When the 128 x BN output tiles cannot fill the SMs (small M, as in
// single-token or short-batch linears), each tile is computed by a cluster of
// `split` CTAs that divide its k-tiles evenly.  Every CTA runs the single-SM
// roles (TMA producer, scale copier, MMA thread) over its k-range into its own
// tensor-memory accumulator; the epilogue warps then park the fp32 partial tile
// in the CTA's (now idle) shared-memory ring, the cluster synchronises, and
// every CTA sums one slice of the tile across all partials through distributed
// shared memory, in rank order (deterministic), scales by alpha and stores it.
// A second cluster barrier keeps every partial alive until all slices are
// read.  Both cluster barriers are reached on every path, errors included.
namespace splitk {

constexpr int kMaxSplit = 8;

template <int BN>
struct Part {
  static constexpr int kStride = BN + 4;                       // floats per row (padding spreads banks)
  static constexpr int kBytes = 128 * kStride * 4;
};

// Called only between the two cluster barriers, which order it against the partials' stores.
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

template <int BN, int FMT, bool BF16>
__global__ void __launch_bounds__(Cfg<BN, FMT, false>::kThreads, 1)
    fp4_gemm_splitk_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                           KernelArgs p, int split) {
  pdl_trigger();
  using C = Cfg<BN, FMT, false>;
  constexpr int S = C::kStages;
  constexpr int APK = C::kApk;
  static_assert(Part<BN>::kBytes <= S * C::kStageBytes, "partial tile must fit in the stage ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * C::kABytes;
  uint8_t* sSFA = sB + S * C::kBBytes;
  uint8_t* sSFB = sSFA + S * C::kSfaBytes;
  float* part = reinterpret_cast<float*>(smem);               // reuses the ring after the last MMA
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + S * C::kSfbBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* drain = bars + 2 * S + 1;
  uint64_t* sfdrain = bars + 2 * S + 2;
  uint64_t* sf_full = bars + 2 * S + 3;
  uint64_t* sf_empty = sf_full + kSfBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + kSfBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = pair::cluster_rank();
  const int tile = (int)(blockIdx.x / (uint32_t)split);
  int mt, nt;
  tile_coords(tile, p.num_m, p.num_n, mt, nt);
  const int nkb = (p.K + BK - 1) / BK;
  const int kb0 = (int)((int64_t)nkb * rank / split), kb1 = (int)((int64_t)nkb * (rank + 1) / split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(tfull), 1);
    mbar_init(smem_u32(drain), 1);
    mbar_init(smem_u32(sfdrain), 1);
    for (uint32_t b = 0; b < kSfBufs; ++b) {
      mbar_init(smem_u32(&sf_full[b]), 1);
      mbar_init(smem_u32(&sf_empty[b]), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();                               // the previous kernel's outputs (our operands) are complete
  bool have_part = false;                                        // this thread wrote its partial rows

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const int rb_total = (p.N + 127) / 128;
      const int rb_here = min(BN / 128, rb_total - nt * (BN / 128));
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_spin(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
          raise_abort(abort_flag, p.error);
          ok = false;
          break;
        }
        const int kvalid = min(BK, p.K - kb * BK);
        const int atoms = (kvalid / FmtTraits<FMT>::kBlock + 3) / 4;
        const uint32_t fb = smem_u32(&full[stage]);
        mbar_expect_tx(fb, (uint32_t)(C::kABytes + C::kBBytes + atoms * 512 * (1 + rb_here)));
        tma_load_2d(smem_u32(sA + stage * C::kABytes), &tmap_a, kb * BK_BYTES, mt * BM, fb);
        tma_load_2d(smem_u32(sB + stage * C::kBBytes), &tmap_b, kb * BK_BYTES, nt * BN, fb);
        bulk_load(smem_u32(sSFA + stage * C::kSfaBytes), p.a_sf + ((size_t)mt * p.g4 + (size_t)kb * APK) * 512,
                  (uint32_t)atoms * 512u, fb);
        for (int rb = 0; rb < rb_here; ++rb)
          bulk_load(smem_u32(sSFB + stage * C::kSfbBytes + rb * APK * 512),
                    p.b_sf + ((size_t)(nt * (BN / 128) + rb) * p.g4 + (size_t)kb * APK) * 512, (uint32_t)atoms * 512u,
                    fb);
        issued |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) {
            volatile int never = 0;
            wait_bounded(smem_u32(&full[s]), (issued_parity >> s) & 1u, &never);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, any_mma = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        const uint32_t n = (uint32_t)(kb - kb0), b = n % kSfBufs, use_b = n / kSfBufs;
        if (!wait_spin(smem_u32(&sf_full[b]), use_b & 1u, abort_flag) ||
            !wait_spin(smem_u32(&full[stage]), phase, abort_flag)) {
          raise_abort(abort_flag, p.error);
          ok = false;
          break;
        }
        tc_fence_after();
        const int kvalid = min(BK, p.K - kb * BK);
        const uint32_t sfa_col = C::kSfBase + b * kSfCols;
        const uint32_t sfb_col = sfa_col + 16u;
        const uint64_t adesc = desc_sw128(smem_u32(sA + stage * C::kABytes));
        const uint64_t bdesc = desc_sw128(smem_u32(sB + stage * C::kBBytes));
        const int nmma = kvalid / 64;
        for (int j = 0; j < nmma; ++j) {
          const uint32_t chunk = FMT == FMT_MX ? (uint32_t)(j >> 1) : (uint32_t)j;
          const uint32_t sf_id = FMT == FMT_MX ? (uint32_t)((j & 1) * 2) : 0u;
          const uint32_t idesc = idesc_base<BN, FMT>() | (sf_id << 29) | (sf_id << 4);
          tc_mma<FMT>(tmem, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, tmem + sfa_col + 4u * chunk,
                      tmem + sfb_col + 4u * chunk * (BN / 128), (kb > kb0 || j > 0) ? 1u : 0u);
          any_mma = true;
        }
        tc_commit(smem_u32(&empty[stage]));
        tc_commit(smem_u32(&sf_empty[b]));
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        tc_commit(smem_u32(tfull));
      } else if (any_mma) {
        tc_commit(smem_u32(drain));
        volatile int never = 0;
        wait_bounded(smem_u32(drain), 0u, &never);
      }
    }
    __syncwarp();
  } else if (warp == C::kSfWarp) {
    // ------------------------------------------------------ scale copier --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, any_cp = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        const uint32_t n = (uint32_t)(kb - kb0), b = n % kSfBufs, use_b = n / kSfBufs;
        if (!wait_spin(smem_u32(&full[stage]), phase, abort_flag) ||
            !wait_spin(smem_u32(&sf_empty[b]), (use_b & 1u) ^ 1u, abort_flag)) {
          raise_abort(abort_flag, p.error);
          ok = false;
          break;
        }
        tc_fence_after();
        const int kvalid = min(BK, p.K - kb * BK);
        const int atoms = (kvalid / FmtTraits<FMT>::kBlock + 3) / 4;
        const uint32_t sfa_col = C::kSfBase + b * kSfCols;
        const uint32_t sfb_col = sfa_col + 16u;
        for (int i = 0; i < atoms; ++i) {
          tc_cp_sf(tmem + sfa_col + 4u * i, desc_sf(smem_u32(sSFA + stage * C::kSfaBytes + i * 512)));
          for (int rb = 0; rb < BN / 128; ++rb)
            tc_cp_sf(tmem + sfb_col + 4u * (i * (BN / 128) + rb),
                     desc_sf(smem_u32(sSFB + stage * C::kSfbBytes + (rb * APK + i) * 512)));
        }
        tc_commit(smem_u32(&sf_full[b]));
        any_cp = true;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok && any_cp) {
        tc_commit(smem_u32(sfdrain));
        volatile int never = 0;
        wait_bounded(smem_u32(sfdrain), 0u, &never);
      }
    }
    __syncwarp();
  } else {
    // -------------------------------------------------- partial tile out --
    const int q = warp & 3;
    const int col0 = ((warp - 2) / 4) * 128;
    int ok = 1;
    if (lane == 0) ok = wait_bounded(smem_u32(tfull), 0u, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok) {
      if (lane == 0) raise_abort(abort_flag, p.error);
    } else {
      tc_fence_after();
      uint32_t r[4][32];
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)col0;
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tbase + (uint32_t)(32 * c), r[c]);
      tmem_ld_wait(r);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // ring bytes last touched by the async proxy
      float4* row = reinterpret_cast<float4*>(part + (size_t)(q * 32 + lane) * Part<BN>::kStride + col0);
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int v = 0; v < 8; ++v)
          row[c * 8 + v] = make_float4(__uint_as_float(r[c][4 * v]), __uint_as_float(r[c][4 * v + 1]),
                                       __uint_as_float(r[c][4 * v + 2]), __uint_as_float(r[c][4 * v + 3]));
      have_part = true;
    }
  }
  (void)have_part;
  tc_fence_before();
  __syncthreads();
  pair::cluster_sync_all();                 // every CTA's partial tile is in its shared memory

  // ------------------------------------------- reduce one slice across ranks --
  {
    const int rows = min(128, p.M - mt * BM);
    constexpr int kC4 = BN / 4;                                   // float4 columns per row
    const int items = rows * kC4;
    const int i0 = (int)((int64_t)items * rank / split), i1 = (int)((int64_t)items * (rank + 1) / split);
    const float alpha = FMT == FMT_NV ? __fmul_rn(*p.a_ts, *p.b_ts) : 1.0f;
    const uint32_t part_base = smem_u32(part);
    for (int it = i0 + (int)threadIdx.x; it < i1; it += (int)blockDim.x) {
      const int row = it / kC4, c4 = it - row * kC4;
      const uint32_t addr = part_base + (uint32_t)((row * Part<BN>::kStride + 4 * c4) * 4);
      float4 v[kMaxSplit];                                       // all remote loads in flight at once
#pragma unroll
      for (int s = 0; s < kMaxSplit; ++s)
        if (s < split) v[s] = ld_cluster_f4(pair::map_rank(addr, (uint32_t)s));
      float4 acc = v[0];
#pragma unroll
      for (int s = 1; s < kMaxSplit; ++s)
        if (s < split) {
          acc.x = __fadd_rn(acc.x, v[s].x);
          acc.y = __fadd_rn(acc.y, v[s].y);
          acc.z = __fadd_rn(acc.z, v[s].z);
          acc.w = __fadd_rn(acc.w, v[s].w);
        }
      const float y4[4] = {__fmul_rn(acc.x, alpha), __fmul_rn(acc.y, alpha), __fmul_rn(acc.z, alpha),
                           __fmul_rn(acc.w, alpha)};
      const int m = mt * BM + row;
      const int n0 = nt * BN + 4 * c4;
      if (BF16) {
        __nv_bfloat16* yr = reinterpret_cast<__nv_bfloat16*>(p.y) + (size_t)m * p.ldy + n0;
        if (p.vec_store && n0 + 4 <= p.N) {
          const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y4[0])) |
                              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y4[1])) << 16);
          const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y4[2])) |
                              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y4[3])) << 16);
          *reinterpret_cast<uint2*>(yr) = make_uint2(lo, hi);
        } else {
          for (int i = 0; i < 4; ++i)
            if (n0 + i < p.N) yr[i] = __float2bfloat16_rn(y4[i]);
        }
      } else {
        float* yr = reinterpret_cast<float*>(p.y) + (size_t)m * p.ldy + n0;
        if (p.vec_store && n0 + 4 <= p.N) {
          *reinterpret_cast<float4*>(yr) = make_float4(y4[0], y4[1], y4[2], y4[3]);
        } else {
          for (int i = 0; i < 4; ++i)
            if (n0 + i < p.N) yr[i] = y4[i];
        }
      }
    }
  }
  pair::cluster_sync_all();                 // no CTA leaves while a peer may still read its partial
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace splitk

// ============================== swap-AB split-K (at most 128 activation rows) ===
// Weight streaming for small M (decode steps and short batches).  The tensor cores compute
// Y^T = W . X^T: 128 rows of the weights W fill the MMA's M dimension and the M <= 128 activation
// rows are its N (BNT = 16, 32, 64 or 128 columns, the block-scaled MMA taking any multiple of 8
// from 8 to 256), so no tensor-core work or shared memory is spent on padding rows of X and each
// stage carries a full 16 KB of W.  Each 128-row weight tile is a cluster of `split` CTAs that
// divide its k-tiles, so every SM streams a disjoint slice of W once.  The roles are the single-SM
// kernel's (TMA producer, scale copier, MMA thread); the four epilogue warps park the fp32 partial
// Y^T tile transposed (one shared-memory row per activation row) in the idle stage ring, and after a
// cluster barrier every CTA sums one slice of it across the cluster through distributed shared
// memory, in rank order (deterministic), scales by alpha and stores rows of Y.  Both cluster
// barriers are reached on every path, errors included.
namespace swapab {

template <int BNT, int FMT>
struct CfgS {
  static constexpr int kApk = FmtTraits<FMT>::kAtomsPerKTile;
  static constexpr int kThreads = 224;                   // producer, MMA, 4 epilogue warps, scale copier
  static constexpr int kSfWarp = 6;
  static constexpr int kWBytes = 128 * BK_BYTES;         // 16 KB of weights per stage
  static constexpr int kXBytes = BNT * BK_BYTES;
  static constexpr int kSfBytes = kApk * 512;            // one 128-row scale block per operand
  static constexpr int kStageBytes = kWBytes + kXBytes + 2 * kSfBytes;
  static constexpr int kStages = kSmemRing / kStageBytes > 8 ? 8 : kSmemRing / kStageBytes;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 1024;
  static constexpr int kPStride = 128 + 4;               // floats per parked row (one activation row)
  static constexpr int kPartBytes = BNT * kPStride * 4;
  static constexpr uint32_t kSfBase = 128;               // scale buffers after the <= 128-column accumulator
  // Twelve 32-column scale buffers (weights' then activations' atoms, <= 16 columns each): a k-tile's
  // MMAs are short here, so the copier may run up to 12 k-tiles ahead of them instead of 4; with 4
  // the copy -> MMA -> release round trip, not the weight stream, set the pace.
  static constexpr uint32_t kSfBufs = 12;
  static constexpr uint32_t kSfCols = 32;
  static_assert(kSfBase + kSfBufs * kSfCols <= kTmemCols, "tensor memory budget");
  static_assert(kPartBytes <= kStages * kStageBytes, "partial tile must fit in the stage ring");
  static_assert(BNT == 16 || BNT == 32 || BNT == 64 || BNT == 128, "activation tile");
};

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

template <int BNT, int FMT, bool BF16>
__global__ void __launch_bounds__(CfgS<BNT, FMT>::kThreads, 1)
    fp4_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                         KernelArgs p, int split) {
  pdl_trigger();
  using C = CfgS<BNT, FMT>;
  constexpr int S = C::kStages;
  constexpr int APK = C::kApk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = smem;
  uint8_t* sX = sW + S * C::kWBytes;
  uint8_t* sSFW = sX + S * C::kXBytes;
  uint8_t* sSFX = sSFW + S * C::kSfBytes;
  float* part = reinterpret_cast<float*>(smem);               // reuses the ring after the last MMA
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFX + S * C::kSfBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* tfull = bars + 2 * S;
  uint64_t* drain = bars + 2 * S + 1;
  uint64_t* sfdrain = bars + 2 * S + 2;
  uint64_t* sf_full = bars + 2 * S + 3;
  uint64_t* sf_empty = sf_full + C::kSfBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_empty + C::kSfBufs);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = split > 1 ? pair::cluster_rank() : 0u;
  const int nt = (int)(blockIdx.x / (uint32_t)split);           // 128-row weight tile
  const int nkb = (p.K + BK - 1) / BK;
  const int kb0 = (int)((int64_t)nkb * rank / split), kb1 = (int)((int64_t)nkb * (rank + 1) / split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(tfull), 1);
    mbar_init(smem_u32(drain), 1);
    mbar_init(smem_u32(sfdrain), 1);
    for (uint32_t b = 0; b < C::kSfBufs; ++b) {
      mbar_init(smem_u32(&sf_full[b]), 1);
      mbar_init(smem_u32(&sf_empty[b]), 1);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();                               // the previous kernel's outputs (our operands) are complete

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_parity = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_spin(smem_u32(&empty[stage]), phase ^ 1u, abort_flag)) {
          raise_abort(abort_flag, p.error);
          ok = false;
          break;
        }
        const int kvalid = min(BK, p.K - kb * BK);
        const int atoms = (kvalid / FmtTraits<FMT>::kBlock + 3) / 4;
        const uint32_t fb = smem_u32(&full[stage]);
        mbar_expect_tx(fb, (uint32_t)(C::kWBytes + C::kXBytes + 2 * atoms * 512));
        tma_load_2d(smem_u32(sW + stage * C::kWBytes), &tmap_w, kb * BK_BYTES, nt * 128, fb);
        tma_load_2d(smem_u32(sX + stage * C::kXBytes), &tmap_x, kb * BK_BYTES, 0, fb);
        bulk_load(smem_u32(sSFW + stage * C::kSfBytes), p.b_sf + ((size_t)nt * p.g4 + (size_t)kb * APK) * 512,
                  (uint32_t)atoms * 512u, fb);
        bulk_load(smem_u32(sSFX + stage * C::kSfBytes), p.a_sf + (size_t)kb * APK * 512, (uint32_t)atoms * 512u, fb);
        issued |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) {
            volatile int never = 0;
            wait_bounded(smem_u32(&full[s]), (issued_parity >> s) & 1u, &never);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, any_mma = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        const uint32_t n = (uint32_t)(kb - kb0), b = n % C::kSfBufs, use_b = n / C::kSfBufs;
        if (!wait_spin(smem_u32(&sf_full[b]), use_b & 1u, abort_flag) ||
            !wait_spin(smem_u32(&full[stage]), phase, abort_flag)) {
          raise_abort(abort_flag, p.error);
          ok = false;
          break;
        }
        tc_fence_after();
        const int kvalid = min(BK, p.K - kb * BK);
        const uint32_t sfw_col = C::kSfBase + b * C::kSfCols;
        const uint32_t sfx_col = sfw_col + 16u;
        const uint64_t wdesc = desc_sw128(smem_u32(sW + stage * C::kWBytes));
        const uint64_t xdesc = desc_sw128(smem_u32(sX + stage * C::kXBytes));
        const int nmma = kvalid / 64;
        for (int j = 0; j < nmma; ++j) {
          const uint32_t chunk = FMT == FMT_MX ? (uint32_t)(j >> 1) : (uint32_t)j;
          const uint32_t sf_id = FMT == FMT_MX ? (uint32_t)((j & 1) * 2) : 0u;
          const uint32_t idesc = idesc_base<BNT, FMT>() | (sf_id << 29) | (sf_id << 4);
          tc_mma<FMT>(tmem, wdesc + (uint64_t)(2 * j), xdesc + (uint64_t)(2 * j), idesc, tmem + sfw_col + 4u * chunk,
                      tmem + sfx_col + 4u * chunk, (kb > kb0 || j > 0) ? 1u : 0u);
          any_mma = true;
        }
        tc_commit(smem_u32(&empty[stage]));
        tc_commit(smem_u32(&sf_empty[b]));
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) {
        tc_commit(smem_u32(tfull));
      } else if (any_mma) {
        tc_commit(smem_u32(drain));
        volatile int never = 0;
        wait_bounded(smem_u32(drain), 0u, &never);
      }
    }
    __syncwarp();
  } else if (warp == C::kSfWarp) {
    // ------------------------------------------------------ scale copier --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, any_cp = false;
      for (int kb = kb0; kb < kb1; ++kb) {
        const uint32_t n = (uint32_t)(kb - kb0), b = n % C::kSfBufs, use_b = n / C::kSfBufs;
        if (!wait_spin(smem_u32(&full[stage]), phase, abort_flag) ||
            !wait_spin(smem_u32(&sf_empty[b]), (use_b & 1u) ^ 1u, abort_flag)) {
          raise_abort(abort_flag, p.error);
          ok = false;
          break;
        }
        tc_fence_after();
        const int kvalid = min(BK, p.K - kb * BK);
        const int atoms = (kvalid / FmtTraits<FMT>::kBlock + 3) / 4;
        const uint32_t sfw_col = C::kSfBase + b * C::kSfCols;
        const uint32_t sfx_col = sfw_col + 16u;
        for (int i = 0; i < atoms; ++i) {
          tc_cp_sf(tmem + sfw_col + 4u * i, desc_sf(smem_u32(sSFW + stage * C::kSfBytes + i * 512)));
          tc_cp_sf(tmem + sfx_col + 4u * i, desc_sf(smem_u32(sSFX + stage * C::kSfBytes + i * 512)));
        }
        tc_commit(smem_u32(&sf_full[b]));
        any_cp = true;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok && any_cp) {
        tc_commit(smem_u32(sfdrain));
        volatile int never = 0;
        wait_bounded(smem_u32(sfdrain), 0u, &never);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------- partial Y^T tile, parked transposed --
    // warp w reads tensor-memory lanes 32*(w%4) .. +31 (weight rows) and all BNT columns
    // (activation rows); activation row m of the partial goes to shared-memory row m.
    const int q = warp & 3;
    int ok = 1;
    if (lane == 0) ok = wait_bounded(smem_u32(tfull), 0u, abort_flag) ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok) {
      if (lane == 0) raise_abort(abort_flag, p.error);
    } else {
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // ring bytes last touched by the async proxy
      float* col = part + q * 32 + lane;
      if (BNT == 16) {
        uint32_t r[16];
        tmem_ld16(tbase, r);
        asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]),
                     "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]),
                     "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
#pragma unroll
        for (int m = 0; m < 16; ++m) col[m * C::kPStride] = __uint_as_float(r[m]);
      } else {
#pragma unroll
        for (int c = 0; c < BNT / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tbase + (uint32_t)(32 * c), r);
          asm volatile("tcgen05.wait::ld.sync.aligned;"
                       : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                         "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                         "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                         "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                         "+r"(r[29]), "+r"(r[30]), "+r"(r[31])::"memory");
#pragma unroll
          for (int i = 0; i < 32; ++i) col[(32 * c + i) * C::kPStride] = __uint_as_float(r[i]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (split > 1) pair::cluster_sync_all();  // every CTA's partial tile is in its shared memory

  // ------------------------------------------- reduce one slice across ranks --
  {
    const int nvalid = min(128, p.N - nt * 128);                  // weight rows of this tile
    const int c4n = (nvalid + 3) / 4;                              // float4 groups per activation row
    const int items = p.M * c4n;
    const int i0 = (int)((int64_t)items * rank / split), i1 = (int)((int64_t)items * (rank + 1) / split);
    const float alpha = FMT == FMT_NV ? __fmul_rn(*p.a_ts, *p.b_ts) : 1.0f;
    const uint32_t part_base = smem_u32(part);
    for (int it = i0 + (int)threadIdx.x; it < i1; it += (int)blockDim.x) {
      const int m = it / c4n, c4 = it - m * c4n;
      const uint32_t addr = part_base + (uint32_t)((m * C::kPStride + 4 * c4) * 4);
      float4 v[splitk::kMaxSplit];                               // all remote loads in flight at once
      if (split == 1) {
        v[0] = *reinterpret_cast<const float4*>(part + m * C::kPStride + 4 * c4);
      } else {
#pragma unroll
        for (int s = 0; s < splitk::kMaxSplit; ++s)
          if (s < split) v[s] = splitk::ld_cluster_f4(pair::map_rank(addr, (uint32_t)s));
      }
      float4 acc = v[0];
#pragma unroll
      for (int s = 1; s < splitk::kMaxSplit; ++s)
        if (s < split) {
          acc.x = __fadd_rn(acc.x, v[s].x);
          acc.y = __fadd_rn(acc.y, v[s].y);
          acc.z = __fadd_rn(acc.z, v[s].z);
          acc.w = __fadd_rn(acc.w, v[s].w);
        }
      const float y4[4] = {__fmul_rn(acc.x, alpha), __fmul_rn(acc.y, alpha), __fmul_rn(acc.z, alpha),
                           __fmul_rn(acc.w, alpha)};
      const int n0 = nt * 128 + 4 * c4;
      if (BF16) {
        __nv_bfloat16* yr = reinterpret_cast<__nv_bfloat16*>(p.y) + (size_t)m * p.ldy + n0;
        if (p.vec_store && n0 + 4 <= p.N) {
          const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y4[0])) |
                              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y4[1])) << 16);
          const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y4[2])) |
                              ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y4[3])) << 16);
          *reinterpret_cast<uint2*>(yr) = make_uint2(lo, hi);
        } else {
          for (int i = 0; i < 4; ++i)
            if (n0 + i < p.N) yr[i] = __float2bfloat16_rn(y4[i]);
        }
      } else {
        float* yr = reinterpret_cast<float*>(p.y) + (size_t)m * p.ldy + n0;
        if (p.vec_store && n0 + 4 <= p.N) {
          *reinterpret_cast<float4*>(yr) = make_float4(y4[0], y4[1], y4[2], y4[3]);
        } else {
          for (int i = 0; i < 4; ++i)
            if (n0 + i < p.N) yr[i] = y4[i];
        }
      }
    }
  }
  if (split > 1) pair::cluster_sync_all();  // no CTA leaves while a peer may still read its partial
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace swapab


// ------------------------------------------------------------------ host ---
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 2-D uint8 view [rows, K/2] of packed codes, box 128 bytes x box_rows, 128B swizzle.
bool make_code_map(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t kbytes, int box_rows) {
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kbytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kbytes};
  cuuint32_t box[2] = {(cuuint32_t)BK_BYTES, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale factors in the tensor-core layout viewed as [atoms, 128] uint32 (512 B
// per atom), box = `box_atoms` consecutive atoms.
bool make_sf_map(CUtensorMap* map, const uint8_t* base, int64_t atoms, int box_atoms) {
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)atoms};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, (cuuint32_t)box_atoms};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 output Y[M, N] (row stride ldy elements) for TMA stores: 32-row x 64-column boxes,
// 128B swizzle.  Returns false (caller falls back to direct stores) when Y is fp32, its rows are
// not 16-byte multiples or its base is not 16-byte aligned.
bool make_y_map(CUtensorMap* map, const GemmParams& gp) {
  if (!gp.y_bf16 || (gp.ldy * 2) % 16 != 0 || (reinterpret_cast<uintptr_t>(gp.y) & 15u) != 0) return false;
  auto enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)gp.N, (cuuint64_t)gp.M};
  cuuint64_t strides[1] = {(cuuint64_t)(gp.ldy * 2)};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, gp.y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The fused-quantization fields of the kernel arguments.
void fill_quant_args(KernelArgs& ka, const GemmParams& gp) {
  ka.q_codes = gp.q_codes;
  ka.q_scales = gp.q_scales;
  ka.q_ts = gp.q_ts;
  ka.q_sf_mma = gp.q_sf_mma;
  const int64_t bs = gp.q_out == 1 ? 32 : 16;
  ka.q_g4 = (int)((gp.N / bs + 3) / 4);
  ka.q_rnd = gp.q_rnd;
  ka.q_mx_thr = gp.q_mx_thr;
  ka.q_keys = fp4dev::philox_keys(gp.q_seed);
}

template <int BN, int FMT, bool BF16, int QO = 0>
cudaError_t run_pair(const GemmParams& gp, int num_sms, cudaStream_t st) {
  using C = pair::Cfg2<BN, FMT>;
  static_assert(C::kStages >= 2, "shared memory too small for two stages");
  auto kernel = pair::fp4_gemm_pair_kernel<BN, FMT, BF16, QO>;
  static const cudaError_t attr =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  const int bs = FmtTraits<FMT>::kBlock;
  const int64_t g4 = (gp.K / bs + 3) / 4;
  CUtensorMap ta, tb, tsa, tsb;
  if (!make_code_map(&ta, gp.a, gp.M, gp.K / 2, 128)) return cudaErrorNotSupported;
  if (!make_code_map(&tb, gp.b, gp.N, gp.K / 2, C::kBRows)) return cudaErrorNotSupported;
  if (!make_sf_map(&tsa, gp.a_sf, (gp.M + 127) / 128 * g4, C::kApk)) return cudaErrorNotSupported;
  if (!make_sf_map(&tsb, gp.b_sf, (gp.N + 127) / 128 * g4, C::kApk)) return cudaErrorNotSupported;
  KernelArgs ka;
  ka.a_sf = gp.a_sf;
  ka.b_sf = gp.b_sf;
  ka.a_ts = gp.a_ts;
  ka.b_ts = gp.b_ts;
  ka.y = gp.y;
  ka.ldy = gp.ldy;
  ka.M = (int)gp.M;
  ka.N = (int)gp.N;
  ka.K = (int)gp.K;
  ka.num_m = (int)((gp.M + 255) / 256);
  ka.num_n = (int)((gp.N + BN - 1) / BN);
  ka.g4 = (int)g4;
  ka.error = gp.error;
  {
    const int64_t esz = gp.y_bf16 ? 2 : 4;
    ka.vec_store = ((gp.ldy * esz) % 32 == 0 && (reinterpret_cast<uintptr_t>(gp.y) & 31u) == 0)   ? 2
                   : ((gp.ldy * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(gp.y) & 15u) == 0) ? 1
                                                                                                   : 0;
  }
  ka.tma_store = 0;
  fill_quant_args(ka, gp);
  const int tiles = ka.num_m * ka.num_n;
  int clusters = num_sms / 2;
  if (tiles < clusters) clusters = tiles;
  return launch_kernel(kernel, dim3(2 * clusters), dim3(C::kThreads), C::kSmemBytes, st, false, 1u, ta, tb, tsa, tsb,
                       ka);
}

template <int BN, int FMT, bool BF16, int QO = 0>
cudaError_t run(const GemmParams& gp, int num_sms, cudaStream_t st) {
  using C = Cfg<BN, FMT>;
  static_assert(C::kStages >= 2, "shared memory too small for two stages");
  static const cudaError_t attr = cudaFuncSetAttribute(fp4_gemm_kernel<BN, FMT, BF16, QO>,
                                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  CUtensorMap ta, tb;
  if (!make_code_map(&ta, gp.a, gp.M, gp.K / 2, BM)) return cudaErrorNotSupported;
  if (!make_code_map(&tb, gp.b, gp.N, gp.K / 2, BN)) return cudaErrorNotSupported;
  KernelArgs ka;
  ka.a_sf = gp.a_sf;
  ka.b_sf = gp.b_sf;
  ka.a_ts = gp.a_ts;
  ka.b_ts = gp.b_ts;
  ka.y = gp.y;
  ka.ldy = gp.ldy;
  ka.M = (int)gp.M;
  ka.N = (int)gp.N;
  ka.K = (int)gp.K;
  ka.num_m = (int)((gp.M + BM - 1) / BM);
  ka.num_n = (int)((gp.N + BN - 1) / BN);
  ka.g4 = (int)((gp.K / FmtTraits<FMT>::kBlock + 3) / 4);
  ka.error = gp.error;
  {
    const int64_t esz = gp.y_bf16 ? 2 : 4;
    ka.vec_store = ((gp.ldy * esz) % 32 == 0 && (reinterpret_cast<uintptr_t>(gp.y) & 31u) == 0)   ? 2
                   : ((gp.ldy * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(gp.y) & 15u) == 0) ? 1
                                                                                                   : 0;
  }
  CUtensorMap ty;
  memset(&ty, 0, sizeof(ty));
  ka.tma_store = QO == 0 && make_y_map(&ty, gp) ? 1 : 0;
  fill_quant_args(ka, gp);
  const int tiles = ka.num_m * ka.num_n;
  const int grid = tiles < num_sms ? tiles : num_sms;
  return launch_kernel(fp4_gemm_kernel<BN, FMT, BF16, QO>, dim3(grid), dim3(C::kThreads), C::kSmemBytes, st, false,
                       1u, ta, tb, ty, ka);
}

// Clusters of `split` CTAs of this kernel that the device can hold at once (0 if unknown).
template <int BN, int FMT, bool BF16>
int splitk_max_clusters(int split) {
  using C = Cfg<BN, FMT, false>;
  static int cache[splitk::kMaxSplit + 1] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (split < 1 || split > splitk::kMaxSplit) return 0;
  if (cache[split] == 0) {
    auto kernel = splitk::fp4_gemm_splitk_kernel<BN, FMT, BF16>;
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)split, 1, 1);
    cfg.blockDim = dim3((unsigned)C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)C::kSmemBytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)split;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess)
      n = -1;
    cache[split] = n;
  }
  return cache[split] > 0 ? cache[split] : 0;
}

template <int BN, int FMT, bool BF16>
cudaError_t run_splitk(const GemmParams& gp, int split, cudaStream_t st) {
  using C = Cfg<BN, FMT, false>;
  auto kernel = splitk::fp4_gemm_splitk_kernel<BN, FMT, BF16>;
  static const cudaError_t attr = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       C::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  CUtensorMap ta, tb;
  if (!make_code_map(&ta, gp.a, gp.M, gp.K / 2, BM)) return cudaErrorNotSupported;
  if (!make_code_map(&tb, gp.b, gp.N, gp.K / 2, BN)) return cudaErrorNotSupported;
  KernelArgs ka;
  ka.a_sf = gp.a_sf;
  ka.b_sf = gp.b_sf;
  ka.a_ts = gp.a_ts;
  ka.b_ts = gp.b_ts;
  ka.y = gp.y;
  ka.ldy = gp.ldy;
  ka.M = (int)gp.M;
  ka.N = (int)gp.N;
  ka.K = (int)gp.K;
  ka.num_m = (int)((gp.M + BM - 1) / BM);
  ka.num_n = (int)((gp.N + BN - 1) / BN);
  ka.g4 = (int)((gp.K / FmtTraits<FMT>::kBlock + 3) / 4);
  ka.error = gp.error;
  {
    const int64_t esz = gp.y_bf16 ? 2 : 4;
    ka.vec_store = ((gp.ldy * esz) % 32 == 0 && (reinterpret_cast<uintptr_t>(gp.y) & 31u) == 0)   ? 2
                   : ((gp.ldy * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(gp.y) & 15u) == 0) ? 1
                                                                                                   : 0;
  }
  ka.tma_store = 0;
  return launch_kernel(kernel, dim3((unsigned)(ka.num_m * ka.num_n * split)), dim3(C::kThreads), C::kSmemBytes, st,
                       false, (unsigned)split, ta, tb, ka, split);
}

// Swap-AB launch: the weights gp.b stream through the MMA's M dimension in 128-row tiles, the
// M <= BNT activation rows gp.a are its N; `split` CTAs (a cluster when > 1) share a tile's k-tiles.
template <int BNT, int FMT, bool BF16>
cudaError_t run_swap(const GemmParams& gp, int split, cudaStream_t st) {
  using C = swapab::CfgS<BNT, FMT>;
  auto kernel = swapab::fp4_gemm_swap_kernel<BNT, FMT, BF16>;
  static const cudaError_t attr = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       C::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  CUtensorMap tw, tx;
  if (!make_code_map(&tw, gp.b, gp.N, gp.K / 2, 128)) return cudaErrorNotSupported;
  if (!make_code_map(&tx, gp.a, gp.M, gp.K / 2, BNT)) return cudaErrorNotSupported;
  KernelArgs ka;
  ka.a_sf = gp.a_sf;
  ka.b_sf = gp.b_sf;
  ka.a_ts = gp.a_ts;
  ka.b_ts = gp.b_ts;
  ka.y = gp.y;
  ka.ldy = gp.ldy;
  ka.M = (int)gp.M;
  ka.N = (int)gp.N;
  ka.K = (int)gp.K;
  ka.num_m = 1;
  ka.num_n = (int)((gp.N + 127) / 128);
  ka.g4 = (int)((gp.K / FmtTraits<FMT>::kBlock + 3) / 4);
  ka.error = gp.error;
  {
    const int64_t esz = gp.y_bf16 ? 2 : 4;
    ka.vec_store = ((gp.ldy * esz) % 32 == 0 && (reinterpret_cast<uintptr_t>(gp.y) & 31u) == 0)   ? 2
                   : ((gp.ldy * esz) % 16 == 0 && (reinterpret_cast<uintptr_t>(gp.y) & 15u) == 0) ? 1
                                                                                                   : 0;
  }
  ka.tma_store = 0;
  return launch_kernel(kernel, dim3((unsigned)(ka.num_n * split)), dim3(C::kThreads), C::kSmemBytes, st, false,
                       (unsigned)split, tw, tx, ka, split);
}

template <int FMT, bool BF16>
cudaError_t dispatch_swap_bnt(const GemmParams& gp, int split, cudaStream_t st) {
  if (gp.M <= 16) return run_swap<16, FMT, BF16>(gp, split, st);
  if (gp.M <= 32) return run_swap<32, FMT, BF16>(gp, split, st);
  if (gp.M <= 64) return run_swap<64, FMT, BF16>(gp, split, st);
  return run_swap<128, FMT, BF16>(gp, split, st);
}

}  // namespace

template <int BN>
static int splitk_fit(const GemmParams& p, int split) {
  if (p.fmt == FMT_MX)
    return p.y_bf16 ? splitk_max_clusters<BN, FMT_MX, true>(split) : splitk_max_clusters<BN, FMT_MX, false>(split);
  return p.y_bf16 ? splitk_max_clusters<BN, FMT_NV, true>(split) : splitk_max_clusters<BN, FMT_NV, false>(split);
}

template <int BN>
static cudaError_t dispatch_splitk(const GemmParams& p, int split, cudaStream_t st) {
  if (p.fmt == FMT_MX)
    return p.y_bf16 ? run_splitk<BN, FMT_MX, true>(p, split, st) : run_splitk<BN, FMT_MX, false>(p, split, st);
  return p.y_bf16 ? run_splitk<BN, FMT_NV, true>(p, split, st) : run_splitk<BN, FMT_NV, false>(p, split, st);
}

template <int BN>
static cudaError_t dispatch_fmt(const GemmParams& p, int num_sms, cudaStream_t st) {
  if (p.fmt == FMT_MX) return p.y_bf16 ? run<BN, FMT_MX, true>(p, num_sms, st) : run<BN, FMT_MX, false>(p, num_sms, st);
  return p.y_bf16 ? run<BN, FMT_NV, true>(p, num_sms, st) : run<BN, FMT_NV, false>(p, num_sms, st);
}

template <int BN>
static cudaError_t dispatch_pair(const GemmParams& p, int num_sms, cudaStream_t st) {
  if (p.fmt == FMT_MX)
    return p.y_bf16 ? run_pair<BN, FMT_MX, true>(p, num_sms, st) : run_pair<BN, FMT_MX, false>(p, num_sms, st);
  return p.y_bf16 ? run_pair<BN, FMT_NV, true>(p, num_sms, st) : run_pair<BN, FMT_NV, false>(p, num_sms, st);
}

// Fused-quantization variants: the pair or single-SM kernel by the same rule as launch_gemm,
// never split-K (its cross-CTA reduction would need its own quantizing epilogue).
template <int QO>
static cudaError_t dispatch_quant(const GemmParams& p, bool pair_tiles, int bn, int num_sms, cudaStream_t st) {
  if (pair_tiles)
    return p.fmt == FMT_MX ? run_pair<256, FMT_MX, false, QO>(p, num_sms, st)
                           : run_pair<256, FMT_NV, false, QO>(p, num_sms, st);
  if (bn == 256)
    return p.fmt == FMT_MX ? run<256, FMT_MX, false, QO>(p, num_sms, st) : run<256, FMT_NV, false, QO>(p, num_sms, st);
  return p.fmt == FMT_MX ? run<128, FMT_MX, false, QO>(p, num_sms, st) : run<128, FMT_NV, false, QO>(p, num_sms, st);
}

cudaError_t launch_gemm(const GemmParams& p, int num_sms, cudaStream_t st) {
  // SM-pair 256 x 256 tiles when K is a multiple of 256 (every scale box then stays inside its row
  // block), long enough (>= 2048) for the single accumulator's epilogue to hide behind the mainloop,
  // and the problem has enough tiles to occupy the SM pairs.  Shorter K runs on single-SM 128 x 256
  // tiles (measured faster at K = 768), N < 256 on 128 x 128 tiles.
  const bool pair_tiles = p.K % 256 == 0 && p.K >= 2048 && p.M >= 256 && p.N >= 256 &&
                          ((p.M + 255) / 256) * ((p.N + 255) / 256) >= num_sms / 2;
  const int bn = p.N >= 256 ? 256 : 128;
  if (p.q_out != 0)
    return p.q_out == 1 ? dispatch_quant<1>(p, pair_tiles, bn, num_sms, st)
                        : dispatch_quant<2>(p, pair_tiles, bn, num_sms, st);
  // at most kGemvMaxM activation rows: the weights stream through the CUDA cores (gemv.cu)
  if (gemv_applies(p)) return launch_gemv(p, num_sms, st);
  const int64_t wtiles = (p.N + 127) / 128, nkb_s = (p.K + BK - 1) / BK;
  if (p.M <= 128 && 2 * wtiles <= num_sms && nkb_s >= 2) {
    // at most 128 activation rows and at most half as many 128-row weight tiles as SMs: swap-AB
    // weight streaming, each tile's k-tiles split over a cluster of 2 to 8 CTAs so that about one
    // CTA runs per SM.  (Both small-M kernels are bound by the tensor-memory scale copies, eight
    // 512-byte atoms per k-tile here; with a single CTA per tile, N > 9472 on 148 SMs, the
    // 128 x 256 split-K tiles below measured faster.)
    int64_t split = std::min<int64_t>(std::min<int64_t>(num_sms / wtiles, splitk::kMaxSplit), nkb_s);
    if (p.fmt == FMT_MX)
      return p.y_bf16 ? dispatch_swap_bnt<FMT_MX, true>(p, (int)split, st)
                      : dispatch_swap_bnt<FMT_MX, false>(p, (int)split, st);
    return p.y_bf16 ? dispatch_swap_bnt<FMT_NV, true>(p, (int)split, st)
                    : dispatch_swap_bnt<FMT_NV, false>(p, (int)split, st);
  }
  if (pair_tiles) return dispatch_pair<256>(p, num_sms, st);
  // Too few output tiles to fill the SMs: split each tile's k-range over a cluster of up to 8 CTAs,
  // as many as keep the launch within one CTA per SM.
  const int64_t tiles = ((p.M + BM - 1) / BM) * ((p.N + bn - 1) / bn);
  const int64_t nkb = (p.K + BK - 1) / BK;
  int64_t split = tiles > 0 ? num_sms / tiles : 1;
  if (split > splitk::kMaxSplit) split = splitk::kMaxSplit;
  if (split > nkb) split = nkb;
  // every cluster must be resident at once: shrink the clusters until the device holds them all
  // (clusters of 8 x 220 KB CTAs need 8 free SMs in one GPC)
  while (split >= 2 &&
         tiles > (bn == 256 ? splitk_fit<256>(p, (int)split) : splitk_fit<128>(p, (int)split)))
    --split;
  if (split >= 2)
    return bn == 256 ? dispatch_splitk<256>(p, (int)split, st) : dispatch_splitk<128>(p, (int)split, st);
  return bn == 256 ? dispatch_fmt<256>(p, num_sms, st) : dispatch_fmt<128>(p, num_sms, st);
}

}  // namespace fp4lib
