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
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
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

// Per-device set-up, keyed by the identifier of the context it was done in: a
// context that was destroyed and created again (cudaDeviceReset) may hold the
// array at another address, so a new context repeats the set-up.
struct Setup {
  unsigned long long ctx_id = 0;   // 0: not done (context identifiers start at 1)
  void* scratch = nullptr;
};

std::mutex g_mutex;
Setup g_setup[kMaxDevices];
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_entry_once;

// Identifier of the calling thread's current context, or 0 when it cannot be read.
unsigned long long current_context_id() {
  std::call_once(g_entry_once, [] {
    void* f0 = nullptr;
    void* f1 = nullptr;
    cudaDriverEntryPointQueryResult q0, q1;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f0, cudaEnableDefault, &q0) == cudaSuccess &&
        q0 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess) {
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f0);
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f1);
    }
  });
  if (g_ctx_current == nullptr || g_ctx_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the array on the current device.  The set-up, done once per device and
// context with that device current, loads the amax kernel and looks up the array's address
// (cudaGetSymbolAddress also loads this file's device code).  Under lazy module loading these two
// steps are where the library's code and the array first take device memory; later calls take
// none.  The host-side symbol is only a stand-in and must never reach a kernel.
fp4_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP4_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  Setup& s = g_setup[dev];
  unsigned long long id = current_context_id();
  if (id == 0 || s.ctx_id != id || s.scratch == nullptr) {
    if (fp4lib::load_amax_fixed_grid_kernel() != cudaSuccess) return FP4_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, fp4_noalloc_scratch) != cudaSuccess || p == nullptr) return FP4_ERR_CUDA;
    if (id == 0) id = current_context_id();   // the runtime calls above made the context current
    s.scratch = p;
    s.ctx_id = id;                             // stays 0 (set-up on every call) if ids are unreadable
  }
  *out = s.scratch;
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
