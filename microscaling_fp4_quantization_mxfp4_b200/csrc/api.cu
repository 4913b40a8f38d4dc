// C ABI of libfp4 (see include/fp4.h for the contract of every entry point).
//
// This layer validates arguments (returning before any CUDA call when they
// are wrong), owns the small per-device scratch buffer, and launches the
// kernels of quantize.cu and gemm.cu on the caller's stream.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include <mutex>

#include "../../include/fp4.h"
#include "fp4_internal.h"

using namespace fp4lib;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  Scratch scratch{};
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];

bool log_enabled() {
  static const bool on = [] {
    const char* e = getenv("FP4_LOG");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}

// Per-device state, created on first use with that device current.
fp4_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FP4_ERR_CUDA;
    void* mem = nullptr;
    const size_t bytes = sizeof(float) * kMaxAmaxBlocks + 2 * sizeof(unsigned) + 256;
    if (cudaMalloc(&mem, bytes) != cudaSuccess) return FP4_ERR_CUDA;
    if (cudaMemset(mem, 0, bytes) != cudaSuccess) return FP4_ERR_CUDA;
    d.scratch.partials = static_cast<float*>(mem);
    d.scratch.counter = reinterpret_cast<unsigned*>(static_cast<char*>(mem) + sizeof(float) * kMaxAmaxBlocks);
    d.scratch.error = d.scratch.counter + 1;
    d.scratch.grid_arrive = d.scratch.counter + 2;
    d.scratch.grid_depart = d.scratch.counter + 3;
    // MSE-searched quantization: its amax, its tensor step's per-CTA sums and completion ticket
    void* mse = nullptr;
    const size_t mse_bytes = sizeof(unsigned long long) * 2 * 17 * kMaxMseCtas + 256;
    if (cudaMalloc(&mse, mse_bytes) != cudaSuccess) return FP4_ERR_CUDA;
    if (cudaMemset(mse, 0, mse_bytes) != cudaSuccess) return FP4_ERR_CUDA;
    d.scratch.mse_partials = static_cast<unsigned long long*>(mse);
    d.scratch.mse_amax = reinterpret_cast<float*>(d.scratch.mse_partials + 2 * 17 * kMaxMseCtas);
    d.scratch.mse_ticket = reinterpret_cast<unsigned*>(d.scratch.mse_amax + 4);
    d.num_sms = sms;
    d.ready = true;
  }
  *out = &d;
  return FP4_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace {

fp4_status check_format(int fmt, int block) {
  if (fmt == FP4_MXFP4 && block == 32) return FP4_OK;
  if (fmt == FP4_NVFP4 && block == 16) return FP4_OK;
  if (fmt != FP4_MXFP4 && fmt != FP4_NVFP4) return FP4_ERR_ARG;
  return FP4_ERR_UNSUPPORTED;
}

fp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FP4_OK : FP4_ERR_CUDA; }

int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Shape/alignment checks shared by the quantizers and the amax pass.
fp4_status check_input(const void* x, int64_t rows, int64_t cols, int64_t ld) {
  if (x == nullptr || rows <= 0 || cols <= 0 || ld < cols) return FP4_ERR_ARG;
  if (cols % 8 != 0 || ld % 8 != 0) return FP4_ERR_SHAPE;
  if (!aligned16(x)) return FP4_ERR_ALIGN;
  if (rows * (cols / 8) >= (int64_t)1 << 32) return FP4_ERR_SHAPE;   // 32-bit chunk indexing
  if (rows >= (int64_t)1 << 31 || cols >= (int64_t)1 << 31) return FP4_ERR_SHAPE;
  return FP4_OK;
}

fp4_status quantize_impl(const void* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int block, int axis,
                         int rnd, uint64_t seed, const float* ts_in, float* ts_out, uint8_t* codes, uint8_t* scales,
                         int sf_layout, int had, float* rotated, cudaStream_t st, void* deq = nullptr,
                         int deq_mode = 0, uint64_t idx_base = 0) {
  int four_six = 0;
  uint32_t mx_thr = 0x800000u;       // OCP exponent rule
  if (fmt == FP4_MXFP4_GS) {         // MXFP4 codes and scales under the MSE-fitted clip threshold
    if (block != 32) return FP4_ERR_UNSUPPORTED;
    fmt = FP4_MXFP4;
    mx_thr = 0x680000u;              // T = 7.25: T/4 = 1 + 0x680000 / 2^23
  }
  if (fmt == FP4_NVFP4_4O6) {        // NVFP4 codes and scales with four-over-six block scales
    if (block != 16) return FP4_ERR_UNSUPPORTED;
    fmt = FP4_NVFP4;
    four_six = 1;
  }
  fp4_status s = check_format(fmt, block);
  if (s != FP4_OK) return s;
  if ((s = check_input(x, rows, cols, ld)) != FP4_OK) return s;
  if (axis != 0 && axis != 1) return FP4_ERR_ARG;
  if (rnd != FP4_RTN && rnd != FP4_SR) return FP4_ERR_ARG;
  if (sf_layout != FP4_SF_ROWMAJOR && sf_layout != FP4_SF_MMA) return FP4_ERR_ARG;
  if (codes == nullptr || scales == nullptr) return FP4_ERR_ARG;
  if (fmt == FP4_NVFP4 && ts_out == nullptr) return FP4_ERR_ARG;
  const int64_t qlen = axis == 1 ? cols : rows;        // length of the quantized axis
  const int64_t orows = axis == 1 ? rows : cols;
  if (qlen % block != 0) return FP4_ERR_SHAPE;
  if (!aligned16(codes)) return FP4_ERR_ALIGN;
  if (deq_mode != 0) {
    if (deq == nullptr) return FP4_ERR_ARG;
    if (axis != 1 || four_six || had != 0) return FP4_ERR_UNSUPPORTED;
    if (!aligned16(deq)) return FP4_ERR_ALIGN;
  }
  if (had != 0) {
    if (had != 16 && had != 32 && had != 64 && had != 128) return FP4_ERR_ARG;
    if (axis != 1 || four_six) return FP4_ERR_UNSUPPORTED;
    if (cols % had != 0) return FP4_ERR_SHAPE;
    if (rotated != nullptr && !aligned16(rotated)) return FP4_ERR_ALIGN;
  }
  DeviceState* d = nullptr;
  if ((s = device_state(&d)) != FP4_OK) return s;
  if (log_enabled())
    fprintf(stderr, "[fp4] quantize rows=%lld cols=%lld ld=%lld fmt=%d axis=%d rnd=%d had=%d sf=%d\n",
            (long long)rows, (long long)cols, (long long)ld, fmt, axis, rnd, had, sf_layout);
  const int64_t groups = qlen / block;
  if (sf_layout == FP4_SF_MMA && axis == 0 && (orows % 128 != 0 || groups % 4 != 0)) {
    // padding bytes of the tensor-core layout must read as scale 0 (the axis-1 kernels write them)
    if (cudaMemsetAsync(scales, 0, (size_t)(round_up(orows, 128) * round_up(groups, 4)), st) != cudaSuccess)
      return FP4_ERR_CUDA;
  }
  QuantizeParams p;
  p.x = x;
  p.rows = rows;
  p.cols = cols;
  p.ld = ld;
  p.fmt = fmt == FP4_MXFP4 ? FMT_MX : FMT_NV;
  p.axis = axis;
  p.rnd = rnd == FP4_RTN ? RND_RTN : RND_SR;
  p.seed = seed;
  p.codes = codes;
  p.scales = scales;
  p.sf_mma = sf_layout == FP4_SF_MMA;
  p.had = had;
  p.rotated = rotated;
  p.error = d->scratch.error;
  p.four_six = four_six;
  p.mx_thr = mx_thr;
  p.deq = deq;
  p.deq_mode = deq_mode;
  p.idx_base = idx_base;
  size_t fused_smem = 0;
  uint32_t fused_tiles = 0;
  if (fmt == FP4_NVFP4 && ts_in == nullptr && axis == 1 && ld == cols &&
      fused_nv_fits(rows, cols, d->num_sms, &fused_smem, &fused_tiles)) {
    // one HBM read: amax and quantize in a single cooperative launch
    return from_cuda(launch_quantize_nv_fused(p, ts_out, d->scratch, d->num_sms, st));
  }
  const float* ts_read = nullptr;
  float* ts_copy = nullptr;
  if (fmt == FP4_NVFP4) {
    if (ts_in != nullptr) {
      ts_read = ts_in;
      ts_copy = (ts_out != ts_in) ? ts_out : nullptr;
    } else {
      cudaError_t e = launch_amax(x, rows, cols, ld, had, 1, ts_out, d->scratch, d->num_sms, st);
      if (e != cudaSuccess) return FP4_ERR_CUDA;
      ts_read = ts_out;
    }
  }
  p.ts = ts_read;
  p.ts_copy_out = ts_copy;
  return from_cuda(launch_quantize(p, d->num_sms, st));
}

}  // namespace

extern "C" {

fp4_status fp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int block, int axis, int rnd,
                        uint64_t seed, const float* tensor_scale_in, float* tensor_scale_out, uint8_t* codes,
                        uint8_t* scales, int sf_layout, void* stream) {
  return quantize_impl(x, rows, cols, ld, fmt, block, axis, rnd, seed, tensor_scale_in, tensor_scale_out, codes,
                       scales, sf_layout, 0, nullptr, static_cast<cudaStream_t>(stream));
}

fp4_status fp4_quantize_shard(const void* x, int64_t rows, int64_t cols, int64_t ld, int64_t first_row, int fmt,
                              int block, int axis, int rnd, uint64_t seed, const float* tensor_scale_in,
                              float* tensor_scale_out, uint8_t* codes, uint8_t* scales, int sf_layout, void* stream) {
  if (first_row < 0 || first_row >= ((int64_t)1 << 40)) return FP4_ERR_ARG;
  const int blk = block > 0 ? block : 1;
  if (axis == 0 && first_row % blk != 0) return FP4_ERR_SHAPE;     // the shard's blocks are the tensor's
  if (cols > 0 && first_row > (((int64_t)1 << 62) / cols)) return FP4_ERR_SHAPE;
  return quantize_impl(x, rows, cols, ld, fmt, block, axis, rnd, seed, tensor_scale_in, tensor_scale_out, codes,
                       scales, sf_layout, 0, nullptr, static_cast<cudaStream_t>(stream), nullptr, 0,
                       (uint64_t)first_row * (uint64_t)(cols > 0 ? cols : 0));
}

fp4_status fp4_hadamard_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int block, int axis,
                                 int rnd, uint64_t seed, const float* tensor_scale_in, float* tensor_scale_out,
                                 uint8_t* codes, uint8_t* scales, int sf_layout, int had_block, float* rotated_out,
                                 void* stream) {
  if (had_block == 0) return FP4_ERR_ARG;
  return quantize_impl(x, rows, cols, ld, fmt, block, axis, rnd, seed, tensor_scale_in, tensor_scale_out, codes,
                       scales, sf_layout, had_block, rotated_out, static_cast<cudaStream_t>(stream));
}

fp4_status fp4_quantize_dequantize(const void* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int block,
                                   int rnd, uint64_t seed, const float* tensor_scale_in, float* tensor_scale_out,
                                   uint8_t* codes, uint8_t* scales, int sf_layout, void* out, int out_dtype,
                                   void* stream) {
  if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_ARG;
  if (out == nullptr) return FP4_ERR_ARG;
  return quantize_impl(x, rows, cols, ld, fmt, block, 1, rnd, seed, tensor_scale_in, tensor_scale_out, codes, scales,
                       sf_layout, 0, nullptr, static_cast<cudaStream_t>(stream), out,
                       out_dtype == FP4_OUT_F32 ? 1 : 2);
}

fp4_status fp4_quantize_2d(const void* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int block, int rnd,
                           uint64_t seed, const float* tensor_scale_in, float* tensor_scale_out, uint8_t* codes,
                           uint8_t* scales, uint8_t* codes_t, uint8_t* scales_t, int sf_layout, void* stream) {
  fp4_status s = check_format(fmt, block);
  if (s != FP4_OK) return s;
  if ((s = check_input(x, rows, cols, ld)) != FP4_OK) return s;
  if (rnd != FP4_RTN && rnd != FP4_SR) return FP4_ERR_ARG;
  if (sf_layout != FP4_SF_ROWMAJOR && sf_layout != FP4_SF_MMA) return FP4_ERR_ARG;
  if (codes == nullptr || scales == nullptr) return FP4_ERR_ARG;
  if ((codes_t == nullptr) != (scales_t == nullptr)) return FP4_ERR_ARG;
  if (fmt == FP4_NVFP4 && tensor_scale_out == nullptr) return FP4_ERR_ARG;
  if (rows % block != 0 || cols % block != 0) return FP4_ERR_SHAPE;
  if (!aligned16(codes) || (codes_t != nullptr && !aligned16(codes_t))) return FP4_ERR_ALIGN;
  DeviceState* d = nullptr;
  if ((s = device_state(&d)) != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (sf_layout == FP4_SF_MMA) {
    // padding bytes of the tensor-core layout must read as scale 0
    const int64_t g = cols / block, gt = rows / block;
    if ((rows % 128 != 0 || g % 4 != 0) &&
        cudaMemsetAsync(scales, 0, (size_t)(round_up(rows, 128) * round_up(g, 4)), st) != cudaSuccess)
      return FP4_ERR_CUDA;
    if (scales_t != nullptr && (cols % 128 != 0 || gt % 4 != 0) &&
        cudaMemsetAsync(scales_t, 0, (size_t)(round_up(cols, 128) * round_up(gt, 4)), st) != cudaSuccess)
      return FP4_ERR_CUDA;
  }
  QuantizeParams p;
  p.x = x;
  p.rows = rows;
  p.cols = cols;
  p.ld = ld;
  p.fmt = fmt == FP4_MXFP4 ? FMT_MX : FMT_NV;
  p.axis = 1;
  p.rnd = rnd == FP4_RTN ? RND_RTN : RND_SR;
  p.seed = seed;
  p.codes = codes;
  p.scales = scales;
  p.sf_mma = sf_layout == FP4_SF_MMA;
  p.had = 0;
  p.rotated = nullptr;
  p.error = d->scratch.error;
  p.ts = nullptr;
  p.ts_copy_out = nullptr;
  if (fmt == FP4_NVFP4) {
    if (tensor_scale_in != nullptr) {
      p.ts = tensor_scale_in;
      p.ts_copy_out = (tensor_scale_out != tensor_scale_in) ? tensor_scale_out : nullptr;
    } else {
      if (launch_amax(x, rows, cols, ld, 0, 1, tensor_scale_out, d->scratch, d->num_sms, st) != cudaSuccess)
        return FP4_ERR_CUDA;
      p.ts = tensor_scale_out;
    }
  }
  return from_cuda(launch_quantize_2d(p, codes_t, scales_t, d->num_sms, st));
}

fp4_status fp4_quantize_mse(const void* x, int64_t rows, int64_t cols, int64_t ld, int fmt, int block, int rnd,
                            uint64_t seed, int iters, float* tensor_scale_out, uint8_t* codes, uint8_t* scales,
                            int sf_layout, void* stream) {
  if (fmt != FP4_NVFP4) return fmt == FP4_MXFP4 ? FP4_ERR_UNSUPPORTED : FP4_ERR_ARG;
  if (block != 16) return FP4_ERR_UNSUPPORTED;
  fp4_status s = check_input(x, rows, cols, ld);
  if (s != FP4_OK) return s;
  if (rnd != FP4_RTN && rnd != FP4_SR) return FP4_ERR_ARG;
  if (iters < 0 || iters > 8) return FP4_ERR_ARG;
  if (sf_layout != FP4_SF_ROWMAJOR && sf_layout != FP4_SF_MMA) return FP4_ERR_ARG;
  if (codes == nullptr || scales == nullptr || tensor_scale_out == nullptr) return FP4_ERR_ARG;
  if (cols % 16 != 0) return FP4_ERR_SHAPE;
  if (!aligned16(codes)) return FP4_ERR_ALIGN;
  DeviceState* d = nullptr;
  if ((s = device_state(&d)) != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t g = cols / 16;
  if (sf_layout == FP4_SF_MMA && (rows % 128 != 0 || g % 4 != 0) &&
      cudaMemsetAsync(scales, 0, (size_t)(round_up(rows, 128) * round_up(g, 4)), st) != cudaSuccess)
    return FP4_ERR_CUDA;
  QuantizeParams p;
  p.x = x;
  p.rows = rows;
  p.cols = cols;
  p.ld = ld;
  p.fmt = FMT_NV;
  p.axis = 1;
  p.rnd = rnd == FP4_RTN ? RND_RTN : RND_SR;
  p.seed = seed;
  p.codes = codes;
  p.scales = scales;
  p.sf_mma = sf_layout == FP4_SF_MMA;
  p.had = 0;
  p.rotated = nullptr;
  p.error = d->scratch.error;
  p.ts = nullptr;
  p.ts_copy_out = nullptr;
  return from_cuda(launch_quantize_mse(p, tensor_scale_out, iters, d->scratch, d->num_sms, st));
}

fp4_status fp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* tensor_scale, int64_t rows,
                          int64_t cols, int fmt, int block, int sf_layout, void* out, int out_dtype, void* stream) {
  fp4_status s = check_format(fmt, block);
  if (s != FP4_OK) return s;
  if (codes == nullptr || scales == nullptr || out == nullptr || rows <= 0 || cols <= 0) return FP4_ERR_ARG;
  if (fmt == FP4_NVFP4 && tensor_scale == nullptr) return FP4_ERR_ARG;
  if (sf_layout != FP4_SF_ROWMAJOR && sf_layout != FP4_SF_MMA) return FP4_ERR_ARG;
  if (out_dtype != FP4_OUT_F32 && out_dtype != FP4_OUT_BF16) return FP4_ERR_ARG;
  if (cols % block != 0) return FP4_ERR_SHAPE;
  if (rows * (cols / 8) >= (int64_t)1 << 32) return FP4_ERR_SHAPE;
  if (!aligned16(codes) || !aligned16(out)) return FP4_ERR_ALIGN;
  DeviceState* d = nullptr;
  if ((s = device_state(&d)) != FP4_OK) return s;
  return from_cuda(launch_dequantize(codes, scales, tensor_scale, rows, cols, fmt == FP4_MXFP4 ? FMT_MX : FMT_NV,
                                     sf_layout == FP4_SF_MMA, out, out_dtype == FP4_OUT_BF16, d->num_sms,
                                     static_cast<cudaStream_t>(stream)));
}

fp4_status fp4_gemm(const uint8_t* a, const uint8_t* a_sf, const float* a_ts, const uint8_t* b, const uint8_t* b_sf,
                    const float* b_ts, int64_t M, int64_t N, int64_t K, int fmt, int block, void* y, int64_t ldy,
                    int y_dtype, void* stream) {
  fp4_status s = check_format(fmt, block);
  if (s != FP4_OK) return s;
  if (a == nullptr || a_sf == nullptr || b == nullptr || b_sf == nullptr || y == nullptr) return FP4_ERR_ARG;
  if (fmt == FP4_NVFP4 && (a_ts == nullptr || b_ts == nullptr)) return FP4_ERR_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || ldy < N) return FP4_ERR_ARG;
  if (y_dtype != FP4_OUT_F32 && y_dtype != FP4_OUT_BF16) return FP4_ERR_ARG;
  if (K % 64 != 0) return FP4_ERR_SHAPE;
  if (M >= (int64_t)1 << 31 || N >= (int64_t)1 << 31 || K >= (int64_t)1 << 31) return FP4_ERR_SHAPE;
  if (!aligned16(a) || !aligned16(b) || !aligned16(a_sf) || !aligned16(b_sf)) return FP4_ERR_ALIGN;
  const uintptr_t esz = y_dtype == FP4_OUT_F32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(y) & (esz - 1)) != 0) return FP4_ERR_ALIGN;
  DeviceState* d = nullptr;
  if ((s = device_state(&d)) != FP4_OK) return s;
  GemmParams p;
  p.a = a;
  p.a_sf = a_sf;
  p.a_ts = a_ts;
  p.b = b;
  p.b_sf = b_sf;
  p.b_ts = b_ts;
  p.M = M;
  p.N = N;
  p.K = K;
  p.fmt = fmt == FP4_MXFP4 ? FMT_MX : FMT_NV;
  p.y = y;
  p.ldy = ldy;
  p.y_bf16 = y_dtype == FP4_OUT_BF16;
  p.error = d->scratch.error;
  cudaError_t e = launch_gemm(p, d->num_sms, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return FP4_ERR_UNSUPPORTED;
  return from_cuda(e);
}

fp4_status fp4_gemm_quantize(const uint8_t* a, const uint8_t* a_sf, const float* a_ts, const uint8_t* b,
                             const uint8_t* b_sf, const float* b_ts, int64_t M, int64_t N, int64_t K, int fmt,
                             int block, int out_fmt, int out_block, int rnd, uint64_t seed, const float* out_tensor_scale,
                             uint8_t* out_codes, uint8_t* out_scales, int out_sf_layout, void* stream) {
  fp4_status s = check_format(fmt, block);
  if (s != FP4_OK) return s;
  uint32_t mx_thr = 0x800000u;
  int q_out = 0;
  if (out_fmt == FP4_MXFP4 || out_fmt == FP4_MXFP4_GS) {
    if (out_block != 32) return FP4_ERR_UNSUPPORTED;
    q_out = 1;
    if (out_fmt == FP4_MXFP4_GS) mx_thr = 0x680000u;
  } else if (out_fmt == FP4_NVFP4) {
    if (out_block != 16) return FP4_ERR_UNSUPPORTED;
    if (out_tensor_scale == nullptr) return FP4_ERR_ARG;
    q_out = 2;
  } else {
    return FP4_ERR_ARG;
  }
  if (a == nullptr || a_sf == nullptr || b == nullptr || b_sf == nullptr) return FP4_ERR_ARG;
  if (out_codes == nullptr || out_scales == nullptr) return FP4_ERR_ARG;
  if (fmt == FP4_NVFP4 && (a_ts == nullptr || b_ts == nullptr)) return FP4_ERR_ARG;
  if (rnd != FP4_RTN && rnd != FP4_SR) return FP4_ERR_ARG;
  if (out_sf_layout != FP4_SF_ROWMAJOR && out_sf_layout != FP4_SF_MMA) return FP4_ERR_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return FP4_ERR_ARG;
  if (K % 64 != 0 || N % 32 != 0) return FP4_ERR_SHAPE;
  if (M >= (int64_t)1 << 31 || N >= (int64_t)1 << 31 || K >= (int64_t)1 << 31) return FP4_ERR_SHAPE;
  if (!aligned16(a) || !aligned16(b) || !aligned16(a_sf) || !aligned16(b_sf) || !aligned16(out_codes))
    return FP4_ERR_ALIGN;
  DeviceState* d = nullptr;
  if ((s = device_state(&d)) != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t g = N / out_block;
  if (out_sf_layout == FP4_SF_MMA && (M % 128 != 0 || g % 4 != 0) &&
      cudaMemsetAsync(out_scales, 0, (size_t)(round_up(M, 128) * round_up(g, 4)), st) != cudaSuccess)
    return FP4_ERR_CUDA;
  GemmParams p;
  p.a = a;
  p.a_sf = a_sf;
  p.a_ts = a_ts;
  p.b = b;
  p.b_sf = b_sf;
  p.b_ts = b_ts;
  p.M = M;
  p.N = N;
  p.K = K;
  p.fmt = fmt == FP4_MXFP4 ? FMT_MX : FMT_NV;
  p.y = nullptr;
  p.ldy = N;
  p.y_bf16 = 0;
  p.error = d->scratch.error;
  p.q_out = q_out;
  p.q_codes = out_codes;
  p.q_scales = out_scales;
  p.q_ts = out_tensor_scale;
  p.q_sf_mma = out_sf_layout == FP4_SF_MMA;
  p.q_rnd = rnd == FP4_SR;
  p.q_seed = seed;
  p.q_mx_thr = mx_thr;
  cudaError_t e = launch_gemm(p, d->num_sms, st);
  if (e == cudaErrorNotSupported) return FP4_ERR_UNSUPPORTED;
  return from_cuda(e);
}

fp4_status fp4_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, float* amax_out, void* stream) {
  fp4_status s = check_input(x, rows, cols, ld);
  if (s != FP4_OK) return s;
  if (amax_out == nullptr) return FP4_ERR_ARG;
  DeviceState* d = nullptr;
  if ((s = device_state(&d)) != FP4_OK) return s;
  return from_cuda(launch_amax(x, rows, cols, ld, 0, 0, amax_out, d->scratch, d->num_sms,
                               static_cast<cudaStream_t>(stream)));
}

fp4_status fp4_nv_tensor_scale(const float* amax, float* tensor_scale_out, void* stream) {
  if (amax == nullptr || tensor_scale_out == nullptr) return FP4_ERR_ARG;
  return from_cuda(launch_nv_tensor_scale(amax, tensor_scale_out, static_cast<cudaStream_t>(stream)));
}

size_t fp4_codes_bytes(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0 || (rows * cols) % 2 != 0) return 0;
  return (size_t)(rows * cols / 2);
}

size_t fp4_scales_bytes(int64_t rows, int64_t cols, int block, int axis, int sf_layout) {
  if (rows <= 0 || cols <= 0 || block <= 0 || (axis != 0 && axis != 1)) return 0;
  const int64_t qlen = axis == 1 ? cols : rows;
  const int64_t orows = axis == 1 ? rows : cols;
  if (qlen % block != 0) return 0;
  const int64_t groups = qlen / block;
  if (sf_layout == FP4_SF_ROWMAJOR) return (size_t)(orows * groups);
  if (sf_layout == FP4_SF_MMA) return (size_t)(round_up(orows, 128) * round_up(groups, 4));
  return 0;
}

fp4_status fp4_check_device_errors(void* stream) {
  DeviceState* d = nullptr;
  fp4_status s = device_state(&d);
  if (s != FP4_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FP4_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, d->scratch.error, sizeof(unsigned), cudaMemcpyDeviceToHost) != cudaSuccess) return FP4_ERR_CUDA;
  if (word != 0) {
    // clear the error word and the single-pass quantizer's barrier counters, which a timed-out
    // launch may have left off zero
    const unsigned zero[3] = {0u, 0u, 0u};
    if (cudaMemcpy(d->scratch.error, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return FP4_ERR_CUDA;
    return FP4_ERR_TIMEOUT;
  }
  return FP4_OK;
}

const char* fp4_status_string(fp4_status status) {
  switch (status) {
    case FP4_OK: return "ok";
    case FP4_ERR_ARG: return "invalid argument";
    case FP4_ERR_SHAPE: return "unsupported shape";
    case FP4_ERR_ALIGN: return "misaligned pointer or leading dimension";
    case FP4_ERR_UNSUPPORTED: return "unsupported format/option combination";
    case FP4_ERR_CUDA: return "CUDA runtime error";
    case FP4_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

}  // extern "C"
