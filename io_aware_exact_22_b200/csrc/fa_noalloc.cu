// fa_noalloc.cu - fa_bwd_noalloc: the backward pass for callers that cannot allocate device
// memory.
//
// fa_bwd needs a caller-provided workspace (the per-tile LSE/D statistics and the fp32 dQ
// accumulator).  Some callers have no way to obtain one: code hosted inside a framework that
// owns every byte of device memory and hands its extensions no allocator, or a hot path whose
// rules forbid calling cudaMalloc (which can synchronise the whole device).  For them, this
// entry point uses a fixed scratch array compiled into the library instead.
//
// The array lives in device memory for as long as the library is loaded, on every GPU where the
// library's device code has been loaded.  All calls share it, on every stream: two calls that
// run at the same time on the GPU (different streams, or different host threads) race on it and
// corrupt each other's results; serialise them.  Each call rewrites every part of the scratch
// it reads before reading it (the first kernel writes all statistics and zeroes the dQ
// accumulator), so whatever an earlier call left behind does not matter.
#include "fa.h"

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace {

constexpr size_t kScratchBytes = FA_BWD_NOALLOC_MAX_SCRATCH_BYTES;

// The scratch itself.  In host code this name is only a stand-in for the device symbol; its
// device address must be obtained with cudaGetSymbolAddress on each device.
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up once per device.
fa_status_t scratch_on_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                      const void* dO, const float* lse, void* dq, void* dk, void* dv,
                                      int B, int H, int N, int d, float scale, int causal,
                                      void* stream) {
  // Sizes beyond the fixed scratch are refused before anything touches the GPU.
  if (B > 0 && H > 0 && N > 0 && d > 0 && fa_bwd_workspace_bytes(B, H, N, d) > kScratchBytes)
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || N <= 0) {  // empty or negative: let fa_bwd give its usual answer
    return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, nullptr, 0, B, H, N, d, scale, causal, stream);
  }
  void* scratch = nullptr;
  const fa_status_t st = scratch_on_current_device(&scratch);
  if (st != FA_OK) return st;
  return fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, scratch, kScratchBytes, B, H, N, d, scale, causal,
                stream);
}
