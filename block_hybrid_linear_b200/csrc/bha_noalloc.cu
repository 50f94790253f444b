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
// Cost: kScratchBytes (32 MiB) of device memory on every GPU where this
// library's device code is loaded, until the process exits.  Under lazy
// module loading (the CUDA default, CUDA_MODULE_LOADING=LAZY) that happens at
// the first call of this entry point on a device; under eager loading
// (CUDA_MODULE_LOADING=EAGER) every context that loads the library holds the
// array from its creation, whether or not this entry point is ever called.
// All calls on a device share that one array: two calls whose kernels overlap
// on the GPU (for example on two streams without ordering between them) race
// on it.  The chunk partials are fully rewritten by each call, so nothing in
// the array needs clearing between calls.
//
// The device address of the array is looked up on the first call made in
// each CUDA context (the first call on a device, and again after
// cudaDeviceReset has replaced the device's context); make that first call
// before any stream capture begins.
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <mutex>

#include "../../include/bha.h"
#include "bha_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB
constexpr int kMaxDevices = 64;

// Chunk partials of the prefill (see bha_state_prefill_workspace_size).
static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

// Per device: the array's address and the context it was looked up in.
struct ScratchEntry {
  std::atomic<void*> ptr{nullptr};
  std::atomic<unsigned long long> ctx_id{0};
};
ScratchEntry g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array in the current context (looked up once
// per context).  In host code the array's name only stands in for the
// symbol; its device address must come from the runtime.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BHA_ERR_CUDA;
  ScratchEntry& e = g_scratch[dev];
  const unsigned long long id = bha::current_context_id();
  void* p = e.ptr.load(std::memory_order_acquire);
  if (p == nullptr || (id != 0 && e.ctx_id.load() != id)) {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    p = e.ptr.load(std::memory_order_relaxed);
    if (p == nullptr || (id != 0 && e.ctx_id.load() != id)) {
      p = nullptr;
      if (cudaGetSymbolAddress(&p, g_prefill_scratch) != cudaSuccess || p == nullptr) {
        cudaGetLastError();   // leave no error behind for a later call to find
        return BHA_ERR_CUDA;
      }
      e.ctx_id.store(bha::current_context_id());
      e.ptr.store(p, std::memory_order_release);
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
