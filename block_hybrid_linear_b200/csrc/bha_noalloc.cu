// bha_state_prefill_noalloc: the prompt prefill for callers that cannot
// allocate device memory.
//
// bha_state_prefill splits long prompts into chunks whose partial states go
// through a caller-provided workspace.  Some callers have no way to provide
// one: a plugin loaded into a host application that owns all device memory,
// a runtime that forbids allocation after start-up (allocation can block or
// fail in the middle of serving), or code running under a memory budget
// enforced by someone else's allocator.  This entry point takes the
// workspace from a fixed-size array that lives in this library's device
// memory instead, so the call itself allocates nothing.
//
// Cost: every GPU that loads this part of the library keeps kScratchBytes
// (32 MiB) of device memory until the process exits.  All calls on a device
// share that one array: two calls whose kernels overlap on the GPU (for
// example on two streams without ordering between them) race on it.  The
// chunk partials are fully rewritten by each call, so nothing in the array
// needs clearing between calls.
//
// The device address of the array is looked up once per device, on the
// first call made with that device current; make that first call before any
// stream capture begins.
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <mutex>

#include "../../include/bha.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB
constexpr int kMaxDevices = 64;

// Chunk partials of the prefill (see bha_state_prefill_workspace_size).
static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

std::atomic<void*> g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device (set-up once per
// device).  In host code the array's name only stands in for the symbol; its
// device address must come from the runtime.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BHA_ERR_CUDA;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess || p == nullptr)
        return BHA_ERR_CUDA;
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return BHA_OK;
}

}  // namespace

extern "C" int bha_state_prefill_noalloc(const void* K, const void* V, int n, int hkv, int T,
                                         int d, bha_dtype dtype, float* S, float* z,
                                         bha_stream_t stream) {
  const size_t need = bha_state_prefill_workspace_size(n, hkv, T, d, dtype);
  if (need > kScratchBytes) return BHA_ERR_WORKSPACE;   // beyond the fixed scratch
  void* ws = nullptr;
  if (need > 0) {
    const int st = scratch_address(&ws);
    if (st != BHA_OK) return st;
  }
  return bha_state_prefill(K, V, n, hkv, T, d, dtype, S, z, ws, need > 0 ? kScratchBytes : 0,
                           stream);
}
