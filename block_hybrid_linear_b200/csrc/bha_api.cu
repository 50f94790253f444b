// C ABI of block-hybrid attention: argument validation, dispatch by dtype,
// workspace queries, the device error word, the tensor-map encoder and the
// host-side block partition.  Every check runs before any launch.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/bha.h"
#include "bha_internal.h"
#include "bha_ptx.cuh"

namespace bha {

// Kernel-reported error (BHA_OK / BHA_ERR_TIMEOUT / BHA_ERR_DEVICE), one per GPU.
__device__ int g_dev_error = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::atomic<bool> ready{false};
  std::atomic<unsigned long long> ctx_id{0};   // context the entry was read in
  int* dev_err = nullptr;
  int sm_count = 0;
  int cc_major = 0;
  int cc_minor = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mutex;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);
PfnCtxGetCurrent g_ctx_current = nullptr;
PfnCtxGetId g_ctx_id = nullptr;
std::once_flag g_ctx_once;

// Per-device entries (the error word's address, the SM count) belong to the
// context they were read in: after cudaDeviceReset the runtime creates a new
// primary context, where the library's device symbols may sit elsewhere.  The
// entry is re-read whenever the current context's ID differs from the one it
// was read in (without the driver's context-ID call, once per device).
int device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BHA_ERR_CUDA;
  DeviceInfo& d = g_devices[dev];
  const unsigned long long id = current_context_id();
  if (!d.ready.load(std::memory_order_acquire) || (id != 0 && d.ctx_id.load() != id)) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!d.ready.load(std::memory_order_relaxed) || (id != 0 && d.ctx_id.load() != id)) {
      d.ready.store(false, std::memory_order_relaxed);
      void* p = nullptr;
      // (also creates the runtime's context on this device if there is none yet)
      if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess) {
        cudaGetLastError();   // leave no error behind for a later call to find
        return BHA_ERR_CUDA;
      }
      if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) !=
              cudaSuccess ||
          cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) !=
              cudaSuccess ||
          cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) !=
              cudaSuccess) {
        cudaGetLastError();
        return BHA_ERR_CUDA;
      }
      d.dev_err = static_cast<int*>(p);
      d.ctx_id.store(current_context_id());
      d.ready.store(true, std::memory_order_release);
    }
  }
  *out = &d;
  return BHA_OK;
}

int make_ctx(bha_stream_t stream, bha_dtype dtype, Ctx* c) {
  DeviceInfo* d = nullptr;
  const int st = device_info(&d);
  if (st != BHA_OK) return st;
  // The tensor-core path is built for sm_100a only.
  if (dtype == BHA_BF16 && d->cc_major != 10) return BHA_ERR_UNSUPPORTED;
  c->stream = reinterpret_cast<cudaStream_t>(stream);
  c->dev_err = d->dev_err;
  c->sm_count = d->sm_count;
  c->dev = static_cast<int>(d - g_devices);
  c->ctx_id = d->ctx_id.load();
  return BHA_OK;
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

bool misaligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) != 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

size_t esize(bha_dtype t) { return t == BHA_BF16 ? 2 : 4; }

bool dtype_ok(bha_dtype t) { return t == BHA_BF16 || t == BHA_F32; }

// d / b support: bf16 needs d = 128; fp32 any d <= 128 with d % 4 == 0.
int check_dims(bha_dtype t, int d, int b_or_1) {
  if (!dtype_ok(t)) return BHA_ERR_UNSUPPORTED;
  if (d < 1 || b_or_1 < 1) return BHA_ERR_INVALID_ARG;
  if (b_or_1 > 64) return BHA_ERR_UNSUPPORTED;
  if (t == BHA_BF16 && d != 128) return BHA_ERR_UNSUPPORTED;
  if (t == BHA_F32 && (d > 128 || d % 4 != 0)) return BHA_ERR_UNSUPPORTED;
  return BHA_OK;
}

// The map must be one of bha_fmap; W is required for the projected map and
// only there.
int check_fmap(bha_fmap fmap, const void* W) {
  const int f = static_cast<int>(fmap);
  if (f != BHA_FMAP_RELU && f != BHA_FMAP_ELU1 && f != BHA_FMAP_RELU_PROJ)
    return BHA_ERR_INVALID_ARG;
  if ((f == BHA_FMAP_RELU_PROJ) != (W != nullptr)) return BHA_ERR_INVALID_ARG;
  if (misaligned(W)) return BHA_ERR_MISALIGNED;
  return BHA_OK;
}

// Bytes of W ([hkv][d][d]); 0 when there is none.
size_t w_bytes(const void* W, int hkv, int d, bha_dtype t) {
  return W == nullptr ? 0 : static_cast<size_t>(hkv) * d * d * esize(t);
}

float resolve_scale(float scale, int d) {
  return scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
}

int launch_status(int rc) {
  if (rc == 0) return BHA_OK;
  if (rc == -4) return BHA_ERR_WORKSPACE;
  return BHA_ERR_CUDA;
}

// Waits on an mbarrier that nothing ever arrives at, with a short limit, to
// exercise the kernels' timeout path: the wait gives up, records
// BHA_ERR_TIMEOUT in the device error word and the kernel returns normally.
__global__ void k_selftest_timeout(int* err, unsigned limit_us) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(smem_u32(&bar), 0, err, &abort_flag, static_cast<uint64_t>(limit_us) * 1000ull);
}

}  // namespace

unsigned long long current_context_id() {
  std::call_once(g_ctx_once, [] {
    void* f0 = nullptr;
    void* f1 = nullptr;
    cudaDriverEntryPointQueryResult q0, q1;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f0, cudaEnableDefault, &q0) == cudaSuccess &&
        q0 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess) {
      g_ctx_current = reinterpret_cast<PfnCtxGetCurrent>(f0);
      g_ctx_id = reinterpret_cast<PfnCtxGetId>(f1);
    }
    cudaGetLastError();
  });
  if (g_ctx_current == nullptr || g_ctx_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id + 1;   // 0 stays "unknown"
}

bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* gaddr,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode == nullptr) return false;
  cuuint64_t gd[5];
  cuuint64_t gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
  const CUresult r =
      g_encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(gaddr), gd, gs, bx,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace bha

using namespace bha;

extern "C" {

const char* bha_status_string(int status) {
  switch (status) {
    case BHA_OK: return "BHA_OK";
    case BHA_ERR_INVALID_ARG: return "BHA_ERR_INVALID_ARG";
    case BHA_ERR_UNSUPPORTED: return "BHA_ERR_UNSUPPORTED";
    case BHA_ERR_MISALIGNED: return "BHA_ERR_MISALIGNED";
    case BHA_ERR_WORKSPACE: return "BHA_ERR_WORKSPACE";
    case BHA_ERR_CUDA: return "BHA_ERR_CUDA";
    case BHA_ERR_TIMEOUT: return "BHA_ERR_TIMEOUT";
    case BHA_ERR_DEVICE: return "BHA_ERR_DEVICE";
    default: return "BHA_ERR_UNKNOWN";
  }
}

int bha_version(void) { return 1; }

int bha_block_partition(int L, int B, int* bounds, int max_bounds) {
  if (L < 0 || B < 1 || bounds == nullptr) return BHA_ERR_INVALID_ARG;
  const long long k = (static_cast<long long>(L) + B - 1) / B;
  if (max_bounds < k + 1) return BHA_ERR_WORKSPACE;
  bounds[0] = 0;
  for (long long i = 1; i <= k; ++i) {
    const long long e = i * B;
    bounds[i] = static_cast<int>(e < L ? e : L);
  }
  return static_cast<int>(k);
}

int bha_device_error(int reset) {
  DeviceInfo* d = nullptr;
  if (device_info(&d) != BHA_OK) return BHA_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return BHA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, d->dev_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return BHA_ERR_CUDA;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpy(d->dev_err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return BHA_ERR_CUDA;
  }
  return v;
}

int bha_selftest_timeout(bha_stream_t stream) {
  DeviceInfo* d = nullptr;
  if (device_info(&d) != BHA_OK) return BHA_ERR_CUDA;
  k_selftest_timeout<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(d->dev_err, 10000u);
  return cudaGetLastError() == cudaSuccess ? BHA_OK : BHA_ERR_CUDA;
}

size_t bha_state_prefill_workspace_size(int n, int hkv, int T, int d, bha_dtype dtype) {
  if (dtype != BHA_BF16 || n <= 0 || hkv <= 0 || T <= 0 || d != 128) return 0;
  return prefill_bf16_workspace(n * hkv, T);
}

int bha_state_prefill(const void* K, const void* V, int n, int hkv, int T, int d,
                      bha_dtype dtype, float* S, float* z, void* workspace,
                      size_t workspace_bytes, bha_stream_t stream) {
  return bha_state_prefill_fm(K, V, n, hkv, T, d, dtype, BHA_FMAP_RELU, nullptr, S, z, workspace,
                              workspace_bytes, stream);
}

}  // extern "C"

namespace {

// bha_state_prefill_fm with optional ragged prompt lengths (device, [n]).
int prefill_impl(const void* K, const void* V, const int* T_lens, int n, int hkv, int T, int d,
                 bha_dtype dtype, bha_fmap fmap, const void* W, float* S, float* z,
                 void* workspace, size_t workspace_bytes, bha_stream_t stream) {
  int st = check_dims(dtype, d, 1);
  if (st != BHA_OK) return st;
  st = check_fmap(fmap, W);
  if (st != BHA_OK) return st;
  if (n < 0 || hkv < 1 || T < 0) return BHA_ERR_INVALID_ARG;
  if (n == 0) return BHA_OK;
  if (S == nullptr || (T > 0 && (K == nullptr || V == nullptr))) return BHA_ERR_INVALID_ARG;
  if (misaligned(K) || misaligned(V) || misaligned(S) || misaligned(z) || misaligned(workspace))
    return BHA_ERR_MISALIGNED;
  const size_t units = static_cast<size_t>(n) * hkv;
  const size_t kv_bytes = units * T * d * esize(dtype);
  const size_t s_bytes = units * d * d * 4, z_bytes = units * d * 4;
  const size_t wb = w_bytes(W, hkv, d, dtype);
  if (overlap(S, s_bytes, K, kv_bytes) || overlap(S, s_bytes, V, kv_bytes) ||
      overlap(z, z_bytes, K, kv_bytes) || overlap(z, z_bytes, V, kv_bytes) ||
      overlap(z, z_bytes, S, s_bytes) || overlap(W, wb, S, s_bytes) || overlap(W, wb, z, z_bytes))
    return BHA_ERR_INVALID_ARG;
  const size_t need = bha_state_prefill_workspace_size(n, hkv, T, d, dtype);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return BHA_ERR_WORKSPACE;
  if (need > 0 && (overlap(workspace, need, S, s_bytes) || overlap(workspace, need, z, z_bytes) ||
                   overlap(workspace, need, K, kv_bytes) || overlap(workspace, need, V, kv_bytes) ||
                   overlap(workspace, need, W, wb) ||
                   overlap(workspace, need, T_lens, static_cast<size_t>(n) * 4)))
    return BHA_ERR_INVALID_ARG;
  if (overlap(T_lens, static_cast<size_t>(n) * 4, S, s_bytes) ||
      overlap(T_lens, static_cast<size_t>(n) * 4, z, z_bytes))
    return BHA_ERR_INVALID_ARG;
  Ctx c;
  st = make_ctx(stream, dtype, &c);
  if (st != BHA_OK) return st;
  if (dtype == BHA_F32)
    return launch_status(launch_prefill_f32(c, static_cast<const float*>(K),
                                            static_cast<const float*>(V), (int)units, T, d, S, z,
                                            fmap, static_cast<const float*>(W), hkv, T_lens));
  return launch_status(launch_prefill_bf16(c, K, V, (int)units, T, S, z, workspace,
                                           workspace_bytes, fmap, W, hkv, T_lens));
}

}  // namespace

extern "C" {

int bha_state_prefill_fm(const void* K, const void* V, int n, int hkv, int T, int d,
                         bha_dtype dtype, bha_fmap fmap, const void* W, float* S, float* z,
                         void* workspace, size_t workspace_bytes, bha_stream_t stream) {
  return prefill_impl(K, V, nullptr, n, hkv, T, d, dtype, fmap, W, S, z, workspace,
                      workspace_bytes, stream);
}

int bha_state_prefill_ragged(const void* K, const void* V, const int* T_lens, int n, int hkv,
                             int Tmax, int d, bha_dtype dtype, bha_fmap fmap, const void* W,
                             float* S, float* z, void* workspace, size_t workspace_bytes,
                             bha_stream_t stream) {
  if (n > 0 && T_lens == nullptr) return BHA_ERR_INVALID_ARG;
  if (misaligned4(T_lens)) return BHA_ERR_MISALIGNED;
  return prefill_impl(K, V, T_lens, n, hkv, Tmax, d, dtype, fmap, W, S, z, workspace,
                      workspace_bytes, stream);
}

int bha_state_commit(const void* Kb, const void* Vb, int n, int hkv, int b, int d,
                     bha_dtype dtype, float* S, float* z, bha_stream_t stream) {
  return bha_state_commit_fm(Kb, Vb, n, hkv, b, d, dtype, BHA_FMAP_RELU, nullptr, S, z, stream);
}

int bha_state_commit_fm(const void* Kb, const void* Vb, int n, int hkv, int b, int d,
                        bha_dtype dtype, bha_fmap fmap, const void* W, float* S, float* z,
                        bha_stream_t stream) {
  int st = check_dims(dtype, d, b);
  if (st != BHA_OK) return st;
  st = check_fmap(fmap, W);
  if (st != BHA_OK) return st;
  if (n < 0 || hkv < 1) return BHA_ERR_INVALID_ARG;
  if (n == 0) return BHA_OK;
  if (Kb == nullptr || Vb == nullptr || S == nullptr) return BHA_ERR_INVALID_ARG;
  if (misaligned(Kb) || misaligned(Vb) || misaligned(S) || misaligned(z))
    return BHA_ERR_MISALIGNED;
  const size_t units = static_cast<size_t>(n) * hkv;
  const size_t kv_bytes = units * b * d * esize(dtype);
  const size_t s_bytes = units * d * d * 4, z_bytes = units * d * 4;
  const size_t wb = w_bytes(W, hkv, d, dtype);
  if (overlap(S, s_bytes, Kb, kv_bytes) || overlap(S, s_bytes, Vb, kv_bytes) ||
      overlap(z, z_bytes, Kb, kv_bytes) || overlap(z, z_bytes, Vb, kv_bytes) ||
      overlap(z, z_bytes, S, s_bytes) || overlap(W, wb, S, s_bytes) || overlap(W, wb, z, z_bytes))
    return BHA_ERR_INVALID_ARG;
  Ctx c;
  st = make_ctx(stream, dtype, &c);
  if (st != BHA_OK) return st;
  if (dtype == BHA_F32)
    return launch_status(launch_commit_f32(c, static_cast<const float*>(Kb),
                                           static_cast<const float*>(Vb), (int)units, b, d, S, z,
                                           fmap, static_cast<const float*>(W), hkv));
  return launch_status(launch_commit_bf16(c, Kb, Vb, (int)units, b, S, z, fmap, W, hkv));
}

int bha_hybrid_step(const void* Qa, const void* Ka, const void* Va, const float* S,
                    const float* z, void* Y, int n, int hq, int hkv, int b, int d, float scale,
                    unsigned flags, bha_dtype dtype, bha_stream_t stream) {
  return bha_hybrid_step_fm(Qa, Ka, Va, S, z, Y, n, hq, hkv, b, d, scale, flags, dtype,
                            BHA_FMAP_RELU, nullptr, stream);
}

int bha_hybrid_step_fm(const void* Qa, const void* Ka, const void* Va, const float* S,
                       const float* z, void* Y, int n, int hq, int hkv, int b, int d, float scale,
                       unsigned flags, bha_dtype dtype, bha_fmap fmap, const void* W,
                       bha_stream_t stream) {
  int st = check_dims(dtype, d, b);
  if (st != BHA_OK) return st;
  st = check_fmap(fmap, W);
  if (st != BHA_OK) return st;
  if (n < 0 || hq < 1 || hkv < 1 || hq % hkv != 0) return BHA_ERR_INVALID_ARG;
  if ((flags & ~BHA_FLAG_SHARED_DENOM) != 0) return BHA_ERR_INVALID_ARG;
  const int shared = (flags & BHA_FLAG_SHARED_DENOM) ? 1 : 0;
  if (n == 0) return BHA_OK;
  if (Qa == nullptr || Ka == nullptr || Va == nullptr || S == nullptr || Y == nullptr)
    return BHA_ERR_INVALID_ARG;
  if (shared && z == nullptr) return BHA_ERR_INVALID_ARG;
  if (misaligned(Qa) || misaligned(Ka) || misaligned(Va) || misaligned(S) || misaligned(z) ||
      misaligned(Y))
    return BHA_ERR_MISALIGNED;
  const size_t es = esize(dtype);
  const size_t q_bytes = static_cast<size_t>(n) * hq * b * d * es;
  const size_t kv_bytes = static_cast<size_t>(n) * hkv * b * d * es;
  const size_t s_bytes = static_cast<size_t>(n) * hkv * d * d * 4;
  const size_t z_bytes = static_cast<size_t>(n) * hkv * d * 4;
  const size_t wb = w_bytes(W, hkv, d, dtype);
  if (overlap(Y, q_bytes, Qa, q_bytes) || overlap(Y, q_bytes, Ka, kv_bytes) ||
      overlap(Y, q_bytes, Va, kv_bytes) || overlap(Y, q_bytes, S, s_bytes) ||
      (shared && overlap(Y, q_bytes, z, z_bytes)) || overlap(Y, q_bytes, W, wb))
    return BHA_ERR_INVALID_ARG;
  Ctx c;
  st = make_ctx(stream, dtype, &c);
  if (st != BHA_OK) return st;
  const float sc = resolve_scale(scale, d);
  if (dtype == BHA_F32)
    return launch_status(launch_step_f32(
        c, static_cast<const float*>(Qa), static_cast<const float*>(Ka),
        static_cast<const float*>(Va), S, shared ? z : nullptr, static_cast<float*>(Y), n, hq,
        hkv, b, d, sc, shared, fmap, static_cast<const float*>(W)));
  return launch_status(launch_step_bf16(c, Qa, Ka, Va, S, shared ? z : nullptr, Y, n, hq, hkv, b,
                                        sc, shared, fmap, W));
}

int bha_hybrid_step_commit(const void* Qa, const void* Ka, const void* Va, float* S, float* z,
                           void* Y, int n, int hq, int hkv, int b, int d, float scale,
                           unsigned flags, bha_dtype dtype, bha_stream_t stream) {
  return bha_hybrid_step_commit_fm(Qa, Ka, Va, S, z, Y, n, hq, hkv, b, d, scale, flags, dtype,
                                   BHA_FMAP_RELU, nullptr, stream);
}

int bha_hybrid_step_commit_fm(const void* Qa, const void* Ka, const void* Va, float* S,
                              float* z, void* Y, int n, int hq, int hkv, int b, int d,
                              float scale, unsigned flags, bha_dtype dtype, bha_fmap fmap,
                              const void* W, bha_stream_t stream) {
  int st = check_dims(dtype, d, b);
  if (st != BHA_OK) return st;
  st = check_fmap(fmap, W);
  if (st != BHA_OK) return st;
  if (n < 0 || hq < 1 || hkv < 1 || hq % hkv != 0) return BHA_ERR_INVALID_ARG;
  if ((flags & ~BHA_FLAG_SHARED_DENOM) != 0) return BHA_ERR_INVALID_ARG;
  const int shared = (flags & BHA_FLAG_SHARED_DENOM) ? 1 : 0;
  if (n == 0) return BHA_OK;
  if (Qa == nullptr || Ka == nullptr || Va == nullptr || S == nullptr || Y == nullptr)
    return BHA_ERR_INVALID_ARG;
  if (shared && z == nullptr) return BHA_ERR_INVALID_ARG;
  if (misaligned(Qa) || misaligned(Ka) || misaligned(Va) || misaligned(S) || misaligned(z) ||
      misaligned(Y))
    return BHA_ERR_MISALIGNED;
  const size_t es = esize(dtype);
  const size_t q_bytes = static_cast<size_t>(n) * hq * b * d * es;
  const size_t kv_bytes = static_cast<size_t>(n) * hkv * b * d * es;
  const size_t s_bytes = static_cast<size_t>(n) * hkv * d * d * 4;
  const size_t z_bytes = static_cast<size_t>(n) * hkv * d * 4;
  if (overlap(Y, q_bytes, Qa, q_bytes) || overlap(Y, q_bytes, Ka, kv_bytes) ||
      overlap(Y, q_bytes, Va, kv_bytes) || overlap(Y, q_bytes, S, s_bytes) ||
      overlap(Y, q_bytes, z, z_bytes) || overlap(S, s_bytes, Qa, q_bytes) ||
      overlap(S, s_bytes, Ka, kv_bytes) || overlap(S, s_bytes, Va, kv_bytes) ||
      overlap(z, z_bytes, Qa, q_bytes) || overlap(z, z_bytes, Ka, kv_bytes) ||
      overlap(z, z_bytes, Va, kv_bytes) || overlap(z, z_bytes, S, s_bytes))
    return BHA_ERR_INVALID_ARG;
  const size_t wb = w_bytes(W, hkv, d, dtype);
  if (overlap(W, wb, Y, q_bytes) || overlap(W, wb, S, s_bytes) || overlap(W, wb, z, z_bytes))
    return BHA_ERR_INVALID_ARG;
  Ctx c;
  st = make_ctx(stream, dtype, &c);
  if (st != BHA_OK) return st;
  const float sc = resolve_scale(scale, d);
  const int units = n * hkv;
  if (dtype == BHA_F32) {
    const float* Wf = static_cast<const float*>(W);
    st = launch_status(launch_step_f32(
        c, static_cast<const float*>(Qa), static_cast<const float*>(Ka),
        static_cast<const float*>(Va), S, shared ? z : nullptr, static_cast<float*>(Y), n, hq,
        hkv, b, d, sc, shared, fmap, Wf));
    if (st != BHA_OK) return st;
    return launch_status(launch_commit_f32(c, static_cast<const float*>(Ka),
                                           static_cast<const float*>(Va), units, b, d, S, z,
                                           fmap, Wf, hkv));
  }
  // one kernel (step, then fold the block in) in the default mode with one
  // 128-row tile per unit
  if (!shared && (hq / hkv) * b <= 128)
    return launch_status(
        launch_step_bf16(c, Qa, Ka, Va, S, nullptr, Y, n, hq, hkv, b, sc, 0, fmap, W, z, 1));
  st = launch_status(launch_step_bf16(c, Qa, Ka, Va, S, shared ? z : nullptr, Y, n, hq, hkv, b,
                                      sc, shared, fmap, W));
  if (st != BHA_OK) return st;
  return launch_status(launch_commit_bf16(c, Ka, Va, units, b, S, z, fmap, W, hkv));
}

size_t bha_prefix_softmax_workspace_size(int n, int hq, int hkv, int b, int d, int P,
                                         bha_dtype dtype) {
  if (dtype != BHA_BF16 || n <= 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || b < 1 || b > 64 ||
      d != 128 || P < 0)
    return 0;
  return prefix_bf16_workspace(n, hq, hkv, b, P);
}

int bha_prefix_softmax(const void* Qa, const void* Kc, const void* Vc, int P, int cap,
                       const void* Ka, const void* Va, void* Y, int n, int hq, int hkv, int b,
                       int d, float scale, bha_dtype dtype, void* workspace,
                       size_t workspace_bytes, bha_stream_t stream) {
  int st = check_dims(dtype, d, b);
  if (st != BHA_OK) return st;
  if (n < 0 || hq < 1 || hkv < 1 || hq % hkv != 0 || P < 0 || cap < P)
    return BHA_ERR_INVALID_ARG;
  if (n == 0) return BHA_OK;
  if (Qa == nullptr || Ka == nullptr || Va == nullptr || Y == nullptr ||
      (P > 0 && (Kc == nullptr || Vc == nullptr)))
    return BHA_ERR_INVALID_ARG;
  if (misaligned(Qa) || misaligned(Kc) || misaligned(Vc) || misaligned(Ka) || misaligned(Va) ||
      misaligned(Y) || misaligned(workspace))
    return BHA_ERR_MISALIGNED;
  const size_t es = esize(dtype);
  const size_t q_bytes = static_cast<size_t>(n) * hq * b * d * es;
  const size_t kv_bytes = static_cast<size_t>(n) * hkv * b * d * es;
  const size_t c_bytes = static_cast<size_t>(n) * hkv * cap * d * es;
  if (overlap(Y, q_bytes, Qa, q_bytes) || overlap(Y, q_bytes, Ka, kv_bytes) ||
      overlap(Y, q_bytes, Va, kv_bytes) || overlap(Y, q_bytes, Kc, c_bytes) ||
      overlap(Y, q_bytes, Vc, c_bytes))
    return BHA_ERR_INVALID_ARG;
  const size_t need = bha_prefix_softmax_workspace_size(n, hq, hkv, b, d, P, dtype);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return BHA_ERR_WORKSPACE;
  if (need > 0 && (overlap(workspace, need, Y, q_bytes) || overlap(workspace, need, Qa, q_bytes) ||
                   overlap(workspace, need, Kc, c_bytes) || overlap(workspace, need, Vc, c_bytes)))
    return BHA_ERR_INVALID_ARG;
  Ctx c;
  st = make_ctx(stream, dtype, &c);
  if (st != BHA_OK) return st;
  const float sc = resolve_scale(scale, d);
  if (dtype == BHA_F32)
    return launch_status(launch_prefix_f32(
        c, static_cast<const float*>(Qa), static_cast<const float*>(Kc),
        static_cast<const float*>(Vc), P, cap, static_cast<const float*>(Ka),
        static_cast<const float*>(Va), static_cast<float*>(Y), n, hq, hkv, b, d, sc));
  return launch_status(launch_prefix_bf16(c, Qa, Kc, Vc, P, cap, Ka, Va, Y, n, hq, hkv, b, sc,
                                          workspace, workspace_bytes));
}

size_t bha_prefix_softmax_reuse_workspace_size(int n, int hq, int hkv, int b, int d, int P,
                                               int k, bha_dtype dtype) {
  if (dtype != BHA_BF16 || n <= 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || b < 1 || b > 64 ||
      d != 128 || P < 0 || k < 0)
    return 0;
  const size_t first = reuse_bf16_workspace(n, hq, hkv, b, P, k, 0);
  const size_t later = reuse_bf16_workspace(n, hq, hkv, b, P, k, 1);
  return first > later ? first : later;
}

int bha_prefix_softmax_reuse(const void* Qa, const void* Qprev, const void* Kc, const void* Vc,
                             int P, int cap, const void* Ka, const void* Va, void* Y,
                             float* O_pre, float* L_pre, int* active, int k, int n, int hq,
                             int hkv, int b, int d, float scale, bha_dtype dtype, void* workspace,
                             size_t workspace_bytes, bha_stream_t stream) {
  int st = check_dims(dtype, d, b);
  if (st != BHA_OK) return st;
  if (n < 0 || hq < 1 || hkv < 1 || hq % hkv != 0 || P < 0 || cap < P || k < 0)
    return BHA_ERR_INVALID_ARG;
  if (static_cast<long long>(hq) * b > 8192) return BHA_ERR_UNSUPPORTED;   // selection scratch
  if (n == 0) return BHA_OK;
  if (Qa == nullptr || Ka == nullptr || Va == nullptr || Y == nullptr || O_pre == nullptr ||
      L_pre == nullptr || (P > 0 && (Kc == nullptr || Vc == nullptr)))
    return BHA_ERR_INVALID_ARG;
  if (misaligned(Qa) || misaligned(Qprev) || misaligned(Kc) || misaligned(Vc) ||
      misaligned(Ka) || misaligned(Va) || misaligned(Y) || misaligned(O_pre) ||
      misaligned(L_pre) || misaligned4(active) || misaligned(workspace))
    return BHA_ERR_MISALIGNED;
  const size_t es = esize(dtype);
  const size_t q_bytes = static_cast<size_t>(n) * hq * b * d * es;
  const size_t kv_bytes = static_cast<size_t>(n) * hkv * b * d * es;
  const size_t c_bytes = static_cast<size_t>(n) * hkv * cap * d * es;
  const size_t o_bytes = static_cast<size_t>(n) * hq * b * d * 4;
  const size_t l_bytes = static_cast<size_t>(n) * hq * b * 4;
  const bool selects = Qprev != nullptr && k > 0 && k < b;
  const size_t a_bytes = selects && active != nullptr ? static_cast<size_t>(n) * k * 4 : 0;
  const void* ins[6] = {Qa, Qprev, Ka, Va, Kc, Vc};
  const size_t in_bytes[6] = {q_bytes, Qprev ? q_bytes : 0, kv_bytes, kv_bytes,
                              P > 0 ? c_bytes : 0, P > 0 ? c_bytes : 0};
  const void* outs[4] = {Y, O_pre, L_pre, a_bytes ? active : nullptr};
  const size_t out_bytes[4] = {q_bytes, o_bytes, l_bytes, a_bytes};
  for (int o = 0; o < 4; ++o) {
    for (int i = 0; i < 6; ++i)
      if (overlap(outs[o], out_bytes[o], ins[i], in_bytes[i])) return BHA_ERR_INVALID_ARG;
    for (int o2 = o + 1; o2 < 4; ++o2)
      if (overlap(outs[o], out_bytes[o], outs[o2], out_bytes[o2])) return BHA_ERR_INVALID_ARG;
  }
  const size_t need = bha_prefix_softmax_reuse_workspace_size(n, hq, hkv, b, d, P, k, dtype);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return BHA_ERR_WORKSPACE;
  if (need > 0) {
    for (int i = 0; i < 6; ++i)
      if (overlap(workspace, need, ins[i], in_bytes[i])) return BHA_ERR_INVALID_ARG;
    for (int o = 0; o < 4; ++o)
      if (overlap(workspace, need, outs[o], out_bytes[o])) return BHA_ERR_INVALID_ARG;
  }
  Ctx c;
  st = make_ctx(stream, dtype, &c);
  if (st != BHA_OK) return st;
  if (dtype == BHA_F32)
    return launch_status(launch_prefix_reuse_f32(
        c, static_cast<const float*>(Qa), static_cast<const float*>(Qprev),
        static_cast<const float*>(Kc), static_cast<const float*>(Vc), P, cap,
        static_cast<const float*>(Ka), static_cast<const float*>(Va), static_cast<float*>(Y),
        O_pre, L_pre, active, k, n, hq, hkv, b, d, resolve_scale(scale, d)));
  return launch_status(launch_prefix_reuse_bf16(c, Qa, Qprev, Kc, Vc, P, cap, Ka, Va, Y, O_pre,
                                                L_pre, active, k, n, hq, hkv, b,
                                                resolve_scale(scale, d), workspace,
                                                workspace_bytes));
}

size_t bha_prefix_softmax_paged_workspace_size(int n, int hq, int hkv, int b, int d,
                                               int max_pages, int page_size, bha_dtype dtype) {
  if (dtype != BHA_BF16 || n <= 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0 || b < 1 || b > 64 ||
      d != 128 || max_pages < 1 || page_size < 1 ||
      static_cast<long long>(max_pages) * page_size > (1 << 30))
    return 0;
  return prefix_paged_bf16_workspace(n, hq, hkv, b, max_pages * page_size);
}

int bha_prefix_softmax_paged(const void* Qa, const void* Kpool, const void* Vpool, int num_pages,
                             int page_size, const int* block_table, int max_pages,
                             const int* P_lens, const void* Ka, const void* Va, void* Y, int n,
                             int hq, int hkv, int b, int d, float scale, bha_dtype dtype,
                             void* workspace, size_t workspace_bytes, bha_stream_t stream) {
  int st = check_dims(dtype, d, b);
  if (st != BHA_OK) return st;
  if (n < 0 || hq < 1 || hkv < 1 || hq % hkv != 0 || num_pages < 1 || max_pages < 1)
    return BHA_ERR_INVALID_ARG;
  int ps_log2 = 0;
  while ((1 << ps_log2) < page_size && ps_log2 < 30) ++ps_log2;
  if (page_size < 16 || page_size > 256 || (1 << ps_log2) != page_size)
    return BHA_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_pages) * page_size > (1 << 30) ||
      static_cast<long long>(num_pages) * hkv > (1ll << 31) - 1)
    return BHA_ERR_UNSUPPORTED;
  if (n == 0) return BHA_OK;
  if (Qa == nullptr || Kpool == nullptr || Vpool == nullptr || block_table == nullptr ||
      P_lens == nullptr || Ka == nullptr || Va == nullptr || Y == nullptr)
    return BHA_ERR_INVALID_ARG;
  if (misaligned(Qa) || misaligned(Kpool) || misaligned(Vpool) || misaligned(Ka) ||
      misaligned(Va) || misaligned(Y) || misaligned(workspace) || misaligned4(block_table) ||
      misaligned4(P_lens))
    return BHA_ERR_MISALIGNED;
  const size_t es = esize(dtype);
  const size_t q_bytes = static_cast<size_t>(n) * hq * b * d * es;
  const size_t kv_bytes = static_cast<size_t>(n) * hkv * b * d * es;
  const size_t pool_bytes = static_cast<size_t>(num_pages) * hkv * page_size * d * es;
  const size_t t_bytes = static_cast<size_t>(n) * max_pages * 4;
  const size_t p_bytes = static_cast<size_t>(n) * 4;
  if (overlap(Y, q_bytes, Qa, q_bytes) || overlap(Y, q_bytes, Ka, kv_bytes) ||
      overlap(Y, q_bytes, Va, kv_bytes) || overlap(Y, q_bytes, Kpool, pool_bytes) ||
      overlap(Y, q_bytes, Vpool, pool_bytes) || overlap(Y, q_bytes, block_table, t_bytes) ||
      overlap(Y, q_bytes, P_lens, p_bytes))
    return BHA_ERR_INVALID_ARG;
  const size_t need =
      bha_prefix_softmax_paged_workspace_size(n, hq, hkv, b, d, max_pages, page_size, dtype);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return BHA_ERR_WORKSPACE;
  if (need > 0 &&
      (overlap(workspace, need, Y, q_bytes) || overlap(workspace, need, Qa, q_bytes) ||
       overlap(workspace, need, Kpool, pool_bytes) || overlap(workspace, need, Vpool, pool_bytes) ||
       overlap(workspace, need, block_table, t_bytes) || overlap(workspace, need, P_lens, p_bytes)))
    return BHA_ERR_INVALID_ARG;
  Ctx c;
  st = make_ctx(stream, dtype, &c);
  if (st != BHA_OK) return st;
  const float sc = resolve_scale(scale, d);
  const PagedCache pg{block_table, P_lens, max_pages, ps_log2, num_pages};
  if (dtype == BHA_F32)
    return launch_status(launch_prefix_paged_f32(
        c, static_cast<const float*>(Qa), static_cast<const float*>(Kpool),
        static_cast<const float*>(Vpool), pg, static_cast<const float*>(Ka),
        static_cast<const float*>(Va), static_cast<float*>(Y), n, hq, hkv, b, d, sc));
  return launch_status(launch_prefix_paged_bf16(c, Qa, Kpool, Vpool, pg, Ka, Va, Y, n, hq, hkv,
                                                b, sc, workspace, workspace_bytes));
}

}  // extern "C"
