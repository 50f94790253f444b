// Internal host-side interface between the C ABI layer and the kernels.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

namespace bha {

struct Ctx {
  cudaStream_t stream;
  int* dev_err;    // device error word of the current device
  int sm_count;    // SMs of the current device
  int dev;         // the current device
  unsigned long long ctx_id;   // its current context (0: not known)
};

// ID of the calling thread's current CUDA context plus one (distinct for
// every context a process creates, so a context re-created after
// cudaDeviceReset gets a new one); 0 when none is current or the driver
// lacks the call.
unsigned long long current_context_id();

// For each device, the context in which a kernel's attributes were last set.
struct Prepared {
  std::atomic<unsigned long long> ctx[64] = {};
};

// Tensor-map encoder fetched from the driver at run time (no libcuda link).
// Returns false if the driver entry point is unavailable or rejects the map.
bool encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* gaddr,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle);

// Sets a kernel's dynamic shared-memory limit and the maximum shared-memory
// carveout once per device and context (`done`), outside any hot path.
template <typename Kernel>
bool prepare_kernel(const Ctx& c, Kernel kern, int smem_bytes, Prepared& done) {
  if (c.dev < 0 || c.dev >= 64) return false;
  const unsigned long long stamp = c.ctx_id == 0 ? 1ull : c.ctx_id;
  if (done.ctx[c.dev].load(std::memory_order_acquire) == stamp) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
      cudaSuccess)
    return false;
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  done.ctx[c.dev].store(stamp, std::memory_order_release);
  return true;
}

// Launches `kern` with programmatic stream serialization: the kernel may be
// scheduled while the previous kernel of the stream finishes; it must call
// pdl_wait() before its first global-memory access.  Returns 0 or -5.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
               cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) return -5;
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

// ---- fp32 reference mode (CUDA cores) ----
// fmap: the bha_fmap value; W: [hkv][d][d] (projected map) or null.
int launch_step_f32(const Ctx& c, const float* Q, const float* K, const float* V,
                    const float* S, const float* z, float* Y, int n, int hq, int hkv, int b,
                    int d, float scale, int shared, int fmap, const float* W);
int launch_commit_f32(const Ctx& c, const float* K, const float* V, int units, int b, int d,
                      float* S, float* z, int fmap, const float* W, int hkv);
int launch_prefill_f32(const Ctx& c, const float* K, const float* V, int units, int T, int d,
                       float* S, float* z, int fmap, const float* W, int hkv,
                       const int* T_lens = nullptr);
int launch_prefix_f32(const Ctx& c, const float* Q, const float* Kc, const float* Vc, int P,
                      int cap, const float* K, const float* V, float* Y, int n, int hq, int hkv,
                      int b, int d, float scale);

// ---- bf16 tensor-core path (tcgen05, d = 128) ----
// fmap: the bha_fmap value; W: [hkv][128][128] bf16 (projected map) or null.
// commit != 0 (default mode, G * b <= 128): also
// S += phi(K)^T V and z += sum phi(k) (z = commit_z, may be null) after the
// step has used S.
int launch_step_bf16(const Ctx& c, const void* Q, const void* K, const void* V, const float* S,
                     const float* z, void* Y, int n, int hq, int hkv, int b, float scale,
                     int shared, int fmap, const void* W, float* commit_z = nullptr,
                     int commit = 0);
int launch_commit_bf16(const Ctx& c, const void* K, const void* V, int units, int b, float* S,
                       float* z, int fmap, const void* W, int hkv);
size_t prefill_bf16_workspace(int units, int T);
// T_lens (device, [n], or null): ragged prompts of at most T tokens each.
int launch_prefill_bf16(const Ctx& c, const void* K, const void* V, int units, int T, float* S,
                        float* z, void* ws, size_t ws_bytes, int fmap, const void* W, int hkv,
                        const int* T_lens = nullptr);
size_t prefix_bf16_workspace(int n, int hq, int hkv, int b, int P);
size_t prefix_paged_bf16_workspace(int n, int hq, int hkv, int b, int Pmax);
// A paged KV cache: request i's token t at row t % 2^ps_log2 of page
// table[i * max_pages + (t >> ps_log2)] of a pool of num_pages pages
// [num_pages][hkv][page_size][d]; P_lens[i] cached tokens (device arrays).
struct PagedCache {
  const int* table;
  const int* P_lens;
  int max_pages;
  int ps_log2;
  int num_pages;
};
int launch_prefix_paged_bf16(const Ctx& c, const void* Q, const void* Kpool, const void* Vpool,
                             const PagedCache& pg, const void* K, const void* V, void* Y, int n,
                             int hq, int hkv, int b, float scale, void* ws, size_t ws_bytes);
int launch_prefix_reuse_f32(const Ctx& c, const float* Q, const float* Qprev, const float* Kc,
                            const float* Vc, int P, int cap, const float* K, const float* V,
                            float* Y, float* O_pre, float* L_pre, int* active, int k, int n,
                            int hq, int hkv, int b, int d, float scale);
int launch_prefix_paged_f32(const Ctx& c, const float* Q, const float* Kpool, const float* Vpool,
                            const PagedCache& pg, const float* K, const float* V, float* Y, int n,
                            int hq, int hkv, int b, int d, float scale);
int launch_prefix_bf16(const Ctx& c, const void* Q, const void* Kc, const void* Vc, int P,
                       int cap, const void* K, const void* V, void* Y, int n, int hq, int hkv,
                       int b, float scale, void* ws, size_t ws_bytes);

// ---- reuse of prefix attention for stable tokens (bf16, d = 128) ----
// Chunking of the reuse path's prefix pass (cache tiles only).
void prefix_only_plan(int units, int rows, int P, int* splits, int* tiles_per);
// The exact path's kernel over the cache alone for `rows` packed query rows
// per unit (Q [units][rows][128]): every chunk's numerators, row max (log2
// units) and row sum to wsO [items][128][128] / wsML [items][256]; P > 0.
int launch_prefix_partials_bf16(const Ctx& c, const void* Q, int rows, const void* Kc,
                                const void* Vc, int P, int cap, int units, int hkv, float scale,
                                float* wsO, float* wsML);
// Block attention of every query row merged with its cached prefix part.
int launch_reuse_block_bf16(const Ctx& c, const void* Q, const void* K, const void* V,
                            const float* O_pre, const float* L_pre, void* Y, int n, int hq,
                            int hkv, int b, float scale);
size_t reuse_bf16_workspace(int n, int hq, int hkv, int b, int P, int k, int have_prev);
int launch_prefix_reuse_bf16(const Ctx& c, const void* Q, const void* Qprev, const void* Kc,
                             const void* Vc, int P, int cap, const void* K, const void* V,
                             void* Y, float* O_pre, float* L_pre, int* active, int k, int n,
                             int hq, int hkv, int b, float scale, void* ws, size_t ws_bytes);

}  // namespace bha
