// Host-side internal interface between the C-ABI layer (api.cu) and the
// kernel launchers (quantize.cu, gemm.cu).  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace fp4lib {

// Programmatic dependent launch.  Every kernel of the library is launched with programmatic
// stream serialization, so its CTAs may be scheduled -- and run their
// shared-memory, barrier and tensor-memory setup -- while the previous kernel in the stream
// drains.  Each kernel calls pdl_wait() before its first global-memory access (that returns once
// the previous grid has completed and its writes are visible) and pdl_trigger() at entry, so that
// the next kernel may be scheduled as soon as every CTA of this one has started.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
#endif

// cudaLaunchKernelEx with the programmatic-serialization attribute, plus optional cooperative
// launch and cluster width.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          bool cooperative, unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[3];
  unsigned n = 0;
  at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cooperative) {
    at[n].id = cudaLaunchAttributeCooperative;
    at[n].val.cooperative = 1;
    ++n;
  }
  if (cluster_x > 1) {
    at[n].id = cudaLaunchAttributeClusterDimension;
    at[n].val.clusterDim.x = cluster_x;
    at[n].val.clusterDim.y = 1;
    at[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// FMT_NV46: NVFP4 with four-over-six block scales (quantizer kernels only; its outputs are NVFP4)
enum { FMT_MX = 0, FMT_NV = 1, FMT_NV46 = 2 };
enum { RND_RTN = 0, RND_SR = 1 };

// Per-device scratch owned by the library (allocated once per device).
struct Scratch {
  float* partials;      // per-CTA maxima of the tensor-amax pass
  unsigned* counter;    // CTA ticket counter of the amax pass (self-resetting)
  unsigned* error;      // device error word set by bounded waits
  unsigned* grid_arrive;  // arrivals at the single-pass NVFP4 quantizer's grid barrier (self-resetting)
  unsigned* grid_depart;  // departures from it; the last CTA out zeroes both
  float* mse_amax;        // MSE-searched quantization: the tensor amax
  unsigned long long* mse_partials;  // its tensor step: [kMaxMseCtas][17][2] per-CTA 128-bit sums
  unsigned* mse_ticket;   // its tensor step's CTA completion counter (self-resetting)
};
constexpr int kMaxAmaxBlocks = 2048;
constexpr int kMaxMseCtas = 1024;

// Unsigned 32-bit division by a runtime constant (round-up multiplier method,
// Hacker's Delight ch. 10): q = (umulhi(n, mul) + n) >> shift for n < 2^32.
struct FastDiv {
  uint32_t d, mul, shift;
};
FastDiv make_fastdiv(uint32_t d);

struct QuantizeParams {
  const void* x;
  int64_t rows, cols, ld;
  int fmt, axis, rnd;
  uint64_t seed;
  const float* ts;        // s_t the kernel reads (NV): caller's or the amax pass output
  float* ts_copy_out;     // if non-null and != ts, block 0 writes s_t here
  uint8_t* codes;
  uint8_t* scales;
  int sf_mma;
  int had;                // 0 or Hadamard block size
  float* rotated;         // optional fp32 dump of the rotated input
  unsigned* error;        // device error word
  int four_six = 0;       // NVFP4: four-over-six block scales
  uint32_t mx_thr = 0x800000u;  // MXFP4 exponent clip threshold as a significand field (0x800000: OCP)
  void* deq = nullptr;    // axis 1: also write the dequantized values [rows, cols] here
  int deq_mode = 0;       // 0: no, 1: fp32, 2: bf16
  uint64_t idx_base = 0;  // row-major index of x's first element in the tensor it is a row shard of
                          // (a multiple of 8; stochastic rounding draws the words of idx_base + index)
};

// amax pass: mode 0 writes max|x| (after rotation when had > 0) to `out`,
// mode 1 writes s_t = amax / 2688 (1.0 for amax == 0).
cudaError_t launch_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, int had, int mode,
                        float* out, const Scratch& s, int num_sms, cudaStream_t st);
// amax pass (mode 0) with a caller-chosen grid; scratch must hold `grid` partials.
cudaError_t launch_amax_fixed_grid(const void* x, int64_t rows, int64_t cols, int64_t ld, float* out,
                                   const Scratch& s, uint32_t grid, cudaStream_t st);
// Loads launch_amax_fixed_grid's kernel onto the current device now (under lazy module loading it
// would otherwise load, and take device memory, at its first launch).
cudaError_t load_amax_fixed_grid_kernel();
cudaError_t launch_nv_tensor_scale(const float* amax, float* out, cudaStream_t st);
cudaError_t launch_quantize(const QuantizeParams& p, int num_sms, cudaStream_t st);
// Square-tile (2-D) quantize along axis 1 (codes/scales) and, when codes_t is not null, the same
// codes transposed with the same tile scales (codes_t/scales_t).  rows, cols multiples of the block.
cudaError_t launch_quantize_2d(const QuantizeParams& p, uint8_t* codes_t, uint8_t* scales_t, int num_sms,
                               cudaStream_t st);
// Single-pass NVFP4 quantize (axis 1, no caller-given s_t) for tensors that fit in shared memory
// across the SMs; fused_nv_fits says whether it applies.  Writes s_t to ts_out.
bool fused_nv_fits(int64_t rows, int64_t cols, int num_sms, size_t* smem, uint32_t* tiles_per_cta);
cudaError_t launch_quantize_nv_fused(const QuantizeParams& p, float* ts_out, const Scratch& s, int num_sms,
                                     cudaStream_t st);
// NVFP4 quantization (axis 1, block 16) with MSE-searched scales: amax pass, `iters` tensor-scale
// steps, then the per-block byte search and the codes (RTN or SR per q.rnd).  Writes s_t to ts_out.
cudaError_t launch_quantize_mse(const QuantizeParams& q, float* ts_out, int iters, const Scratch& s, int num_sms,
                                cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* ts, int64_t rows,
                              int64_t cols, int fmt, int sf_mma, void* out, int out_bf16, int num_sms,
                              cudaStream_t st);

struct GemmParams {
  const uint8_t* a;
  const uint8_t* a_sf;
  const float* a_ts;
  const uint8_t* b;
  const uint8_t* b_sf;
  const float* b_ts;
  int64_t M, N, K;
  int fmt;
  void* y;
  int64_t ldy;
  int y_bf16;
  unsigned* error;
  // fused quantization of Y along its rows instead of storing it: 0 (store Y), 1 (MXFP4 codes),
  // 2 (NVFP4 codes under the tensor scale q_ts)
  int q_out = 0;
  uint8_t* q_codes = nullptr;
  uint8_t* q_scales = nullptr;
  const float* q_ts = nullptr;
  int q_sf_mma = 0;
  int q_rnd = 0;
  uint64_t q_seed = 0;
  uint32_t q_mx_thr = 0x800000u;
};
// Returns cudaErrorNotSupported if the driver entry point for tensor maps is missing.
cudaError_t launch_gemm(const GemmParams& p, int num_sms, cudaStream_t st);

// CUDA-core GEMM for at most kGemvMaxM activation rows (gemv.cu): taken by launch_gemm when
// gemv_applies (plain Y output, the converted activations fit kGemvMaxSmem of shared memory).
// One row: measured faster than the tensor-core swap-AB kernel for every Llama-7B shape (NVFP4
// 4096 x 4096: 7.0 -> 5.0 us, MXFP4 6.6 -> 4.1 us); two or more rows were not.
constexpr int64_t kGemvMaxM = 1;
constexpr size_t kGemvMaxSmem = 160 * 1024;
bool gemv_applies(const GemmParams& p);
cudaError_t launch_gemv(const GemmParams& p, int num_sms, cudaStream_t st);

}  // namespace fp4lib
