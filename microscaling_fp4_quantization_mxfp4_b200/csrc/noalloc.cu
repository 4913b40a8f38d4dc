// fp4_amax_noalloc: the tensor amax without any device allocation.
//
// fp4_amax keeps its per-CTA partial maxima in a scratch buffer that the
// library cudaMallocs on first use.  Some callers cannot let that happen:
// a process whose caching allocator already holds all free device memory (a
// late cudaMalloc fails or fragments the pool), a latency-critical caller that
// cannot absorb the device-wide synchronization a cudaMalloc may trigger, or
// code running inside an allocator callback, where calling back into the CUDA
// allocator is not allowed.  For them this entry point keeps its scratch in a
// fixed array compiled into the library instead.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/fp4.h"
#include "fp4_internal.h"

namespace {

// One CTA covers this many 256-element warp tiles, so the grid (and the
// number of partial maxima) grows with the input: at most kMaxCtas CTAs.
constexpr uint32_t kTilesPerCta = 32;                       // 8192 elements per CTA
constexpr uint32_t kMaxCtas = 8192;                         // -> at most 2^26 elements per call
constexpr size_t kCounterOffset = sizeof(float) * kMaxCtas; // 32768
constexpr size_t kScratchBytes = kCounterOffset + 256;      // 33,024 bytes in total

// The scratch: kMaxCtas partial maxima followed by the CTA ticket counter.
// Every GPU that loads libfp4 holds these bytes until the process exits.
static __device__ __align__(256) unsigned char fp4_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per
// device (the host-side symbol is only a stand-in and must never reach a kernel).
fp4_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, fp4_noalloc_scratch) != cudaSuccess || p == nullptr) return FP4_ERR_CUDA;
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return FP4_OK;
}

}  // namespace

extern "C" fp4_status fp4_amax_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld, float* amax_out,
                                       void* stream) {
  if (x == nullptr || amax_out == nullptr || rows <= 0 || cols <= 0 || ld < cols) return FP4_ERR_ARG;
  if (cols % 8 != 0 || ld % 8 != 0) return FP4_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) != 0) return FP4_ERR_ALIGN;
  if (rows > ((int64_t)1 << 26) || cols > ((int64_t)1 << 26)) return FP4_ERR_SHAPE;
  const int64_t tiles = (rows * (cols / 8) + 31) / 32;
  const int64_t ctas = (tiles + kTilesPerCta - 1) / kTilesPerCta;
  if (ctas > (int64_t)kMaxCtas) return FP4_ERR_SHAPE;      // more than 2^26 elements: scratch too small
  void* base = nullptr;
  fp4_status s = scratch_address(&base);
  if (s != FP4_OK) return s;
  fp4lib::Scratch sc;
  sc.partials = static_cast<float*>(base);
  sc.counter = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(base) + kCounterOffset);
  sc.error = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the ticket counter must start at zero; the partials are written before they are read
  if (cudaMemsetAsync(sc.counter, 0, sizeof(unsigned), st) != cudaSuccess) return FP4_ERR_CUDA;
  return fp4lib::launch_amax_fixed_grid(x, rows, cols, ld, amax_out, sc, (uint32_t)ctas, st) == cudaSuccess
             ? FP4_OK
             : FP4_ERR_CUDA;
}
