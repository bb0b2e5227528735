// Workspace-free variant of the fused forward (pa_attend_noalloc).
//
// Some callers cannot allocate device memory at the point where they run
// attention: code inside a memory pool that forbids further cudaMalloc, an
// allocator-free runtime, or a framework hook that must not touch the caching
// allocator.  For them the workspace (plan tables, fp32 partial rows, arrival
// counters and the status word) lives in one file-scope device array instead
// of a caller-provided buffer.  Every GPU that loads the library keeps this
// array (kScratchBytes) for the life of the process.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "plan.h"

namespace {

constexpr size_t kScratchBytes = size_t(24) << 20;  // 24 MiB

static __device__ __align__(256) uint8_t g_pa_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[64] = {};

// Device address of g_pa_scratch on the current device.  The host-side name of
// the array is not a device address; the first call on each device looks the
// address up (with that device current) and caches it.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pa_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

void* pa_noalloc_scratch() { return scratch_address(); }

extern "C" pa_status pa_attend_noalloc(const pa_plan* plan, const void* q, const void* k_pool, const void* v_pool,
                                       void* out, float* lse, void* stream) {
  if (!plan || !q || !k_pool || !v_pool || !out) return PA_ERR_INVALID;
  if (plan->hdr.workspace_bytes > kScratchBytes) return PA_ERR_NOMEM;
  void* ws = scratch_address();
  if (!ws) return PA_ERR_CUDA;
  // The plan image (with the status word and the arrival counters at zero) is
  // copied straight from the plan's host memory: no pinned staging buffer is
  // taken, so nothing is allocated by this call.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(ws, plan->image.data(), plan->image.size, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return PA_ERR_CUDA;
  plan->dev_image = nullptr;  // the launches read this copy
  return pa_attend_ws(plan, q, k_pool, v_pool, ws, out, lse, stream);
}
