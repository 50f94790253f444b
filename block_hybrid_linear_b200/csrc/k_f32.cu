// fp32 reference-mode kernels (CUDA cores, FFMA): the same operations as the
// bf16 tensor-core path with fp32 Q/K/V/Y, any d <= 128 (d % 4 == 0) and
// b <= 64.  Used for the worked example (d = 16) and tight-tolerance checks.
// Simple one-row-at-a-time structure; not a performance path.  Feature
// maps: 0 ReLU, 1 elu + 1, 2 ReLU(x W_g) with W [hkv][d][d] fp32.
#include <cuda_runtime.h>
#include <math.h>

#include "bha_internal.h"

namespace bha {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ float relu(float x) { return x > 0.f ? x : 0.f; }

// Feature r of phi(x) for one d-vector x; Wg = W[g] for the projected map.
__device__ __forceinline__ float phi_at(const float* x, int r, int d, int fmap, const float* Wg) {
  if (fmap == 2) {
    float acc = 0.f;
    for (int i = 0; i < d; ++i) acc = fmaf(x[i], Wg[(size_t)i * d + r], acc);
    return relu(acc);
  }
  const float v = x[r];
  if (fmap == 1) return v > 0.f ? v + 1.f : expf(v);
  return relu(v);
}

__device__ float block_reduce_max(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kThreads / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

__device__ float block_reduce_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x / 32, l = threadIdx.x % 32;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = 0.f;
  for (int i = 0; i < kThreads / 32; ++i) r += red[i];
  return r;
}

// One CTA per (request, query head).  Row by row: scores against the b block
// keys, softmax, then each thread produces one output column
//   y[c] = sum_j p_j v_j[c] + sum_r phi(q)_r S[r][c]      (default)
//   y[c] = (sum_j e_j v_j[c] + e^{-m} lin[c]) / (l + e^{-m} phi(q).z)  (shared)
__global__ void __launch_bounds__(kThreads) k_step_f32(const float* __restrict__ Q,
                                                       const float* __restrict__ K,
                                                       const float* __restrict__ V,
                                                       const float* __restrict__ S,
                                                       const float* __restrict__ z,
                                                       float* __restrict__ Y, int hq, int hkv,
                                                       int b, int d, float scale, int shared,
                                                       int fmap, const float* __restrict__ W) {
  extern __shared__ float sm[];
  float* sK = sm;              // [b][d]
  float* sV = sK + b * d;      // [b][d]
  float* sq = sV + b * d;      // [d]
  float* sp = sq + d;          // [b]
  float* sphi = sp + b;        // [d]  phi(q)
  __shared__ float red[kThreads / 32];

  const int nh = blockIdx.x;
  const int ni = nh / hq, h = nh % hq, g = h / (hq / hkv);
  const size_t kv_off = ((size_t)ni * hkv + g) * b * d;
  for (int e = threadIdx.x; e < b * d; e += kThreads) {
    sK[e] = K[kv_off + e];
    sV[e] = V[kv_off + e];
  }
  const float* Sg = S + ((size_t)ni * hkv + g) * d * d;
  const float* zg = z ? z + ((size_t)ni * hkv + g) * d : nullptr;
  const float* Wg = W ? W + (size_t)g * d * d : nullptr;
  __syncthreads();

  for (int i = 0; i < b; ++i) {
    const size_t row = (((size_t)ni * hq + h) * b + i) * d;
    for (int c = threadIdx.x; c < d; c += kThreads) sq[c] = Q[row + c];
    __syncthreads();
    for (int c = threadIdx.x; c < d; c += kThreads) sphi[c] = phi_at(sq, c, d, fmap, Wg);
    float s = -INFINITY;
    if (threadIdx.x < b) {
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(sq[c], sK[threadIdx.x * d + c], acc);
      s = acc * scale;
    }
    const float m = block_reduce_max(s, red);
    const float e = threadIdx.x < b ? expf(s - m) : 0.f;
    const float l = block_reduce_sum(e, red);
    if (threadIdx.x < b) sp[threadIdx.x] = e;
    float qz = 0.f;
    if (shared) {
      float part = 0.f;
      for (int r = threadIdx.x; r < d; r += kThreads) part = fmaf(sphi[r], zg[r], part);
      qz = block_reduce_sum(part, red);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < d; c += kThreads) {
      float soft = 0.f;
      for (int j = 0; j < b; ++j) soft = fmaf(sp[j], sV[j * d + c], soft);
      float lin = 0.f;
      for (int r = 0; r < d; ++r) lin = fmaf(sphi[r], Sg[(size_t)r * d + c], lin);
      float y;
      if (!shared) {
        y = soft / l + lin;
      } else {
        const float em = expf(-m);
        y = (soft + em * lin) / (l + em * qz);
      }
      Y[row + c] = y;
    }
    __syncthreads();
  }
}

// S[u][r][c] (+)= sum_t phi(k_t)[r] V[u][t][c];  z[u][r] (+)= sum_t phi(k_t)[r].
// One thread per (r, c) state element; accumulate != 0 adds to S (commit),
// otherwise overwrites (prefill).
__global__ void __launch_bounds__(kThreads) k_state_f32(const float* __restrict__ K,
                                                        const float* __restrict__ V, int T,
                                                        int d, float* __restrict__ S,
                                                        float* __restrict__ z, int accumulate,
                                                        int fmap, const float* __restrict__ W,
                                                        int hkv, const int* __restrict__ T_lens) {
  const int u = blockIdx.y;
  const int e = blockIdx.x * kThreads + threadIdx.x;
  const float* Ku = K + (size_t)u * T * d;
  const float* Vu = V + (size_t)u * T * d;
  // ragged prompts: this request's own length; rows past it are padding
  const int Tu = T_lens ? min(max(T_lens[u / hkv], 0), T) : T;
  const float* Wg = W ? W + (size_t)(u % hkv) * d * d : nullptr;
  if (e < d * d) {
    const int r = e / d, c = e % d;
    float acc = 0.f;
    for (int t = 0; t < Tu; ++t)
      acc = fmaf(phi_at(Ku + (size_t)t * d, r, d, fmap, Wg), Vu[(size_t)t * d + c], acc);
    float* dst = S + (size_t)u * d * d + e;
    *dst = accumulate ? *dst + acc : acc;
  }
  if (z && e < d) {
    float acc = 0.f;
    for (int t = 0; t < Tu; ++t) acc += phi_at(Ku + (size_t)t * d, e, d, fmap, Wg);
    float* dst = z + (size_t)u * d + e;
    *dst = accumulate ? *dst + acc : acc;
  }
}

// A paged cache for the exact path (null table: contiguous [n][hkv][cap][d]).
struct PagedF32 {
  const int* table;   // [n][max_pages]
  const int* P_lens;  // [n]
  int max_pages;
  int ps_log2;
  int num_pages;      // page numbers outside [0, num_pages) read as zero rows
};

// Exact softmax over [cache[0:P] || block]: one CTA per (request, head, row);
// keys are scored 128 at a time with an online max / sum rescale.  Paged:
// request ni's cache is its first P_lens[ni] tokens, token j at row
// j % page_size of page table[ni][j / page_size] of [pages][hkv][page_size][d].
__global__ void __launch_bounds__(kThreads) k_prefix_f32(
    const float* __restrict__ Q, const float* __restrict__ Kc, const float* __restrict__ Vc,
    int P, int cap, const float* __restrict__ K, const float* __restrict__ V,
    float* __restrict__ Y, int hq, int hkv, int b, int d, float scale, PagedF32 pg) {
  extern __shared__ float sm[];
  float* sq = sm;           // [d]
  float* se = sq + d;       // [kThreads]
  float* acc = se + kThreads;  // [d]
  __shared__ float red[kThreads / 32];

  const int id = blockIdx.x;
  const int i = id % b, nh = id / b;
  const int ni = nh / hq, h = nh % hq, g = h / (hq / hkv);
  const size_t row = (((size_t)ni * hq + h) * b + i) * d;
  const float* Kcg = pg.table ? Kc : Kc + ((size_t)ni * hkv + g) * cap * d;
  const float* Vcg = pg.table ? Vc : Vc + ((size_t)ni * hkv + g) * cap * d;
  if (pg.table) P = min(max(pg.P_lens[ni], 0), pg.max_pages << pg.ps_log2);
  const int ps_mask = (1 << pg.ps_log2) - 1;
  __shared__ float zrow[128];   // the row of a page number out of range
  for (int c = threadIdx.x; c < d; c += kThreads) zrow[c] = 0.f;
  // cached token jj's row of the cache at cb (K or V)
  auto cache_row = [&](const float* cb, int jj) -> const float* {
    if (!pg.table) return cb + (size_t)jj * d;
    const int page = pg.table[(size_t)ni * pg.max_pages + (jj >> pg.ps_log2)];
    if (page < 0 || page >= pg.num_pages) return zrow;
    return cb + (((size_t)page * hkv + g) * ((size_t)ps_mask + 1) + (jj & ps_mask)) * d;
  };
  const float* Kg = K + ((size_t)ni * hkv + g) * b * d;
  const float* Vg = V + ((size_t)ni * hkv + g) * b * d;
  for (int c = threadIdx.x; c < d; c += kThreads) {
    sq[c] = Q[row + c];
    acc[c] = 0.f;
  }
  __syncthreads();
  const int L = P + b;
  float m_run = -INFINITY, l_run = 0.f;
  for (int j0 = 0; j0 < L; j0 += kThreads) {
    const int j = j0 + threadIdx.x;
    float s = -INFINITY;
    if (j < L) {
      const float* k = j < P ? cache_row(Kcg, j) : Kg + (size_t)(j - P) * d;
      float a = 0.f;
      for (int c = 0; c < d; ++c) a = fmaf(sq[c], k[c], a);
      s = a * scale;
    }
    const float m_new = fmaxf(m_run, block_reduce_max(s, red));
    const float e = j < L ? expf(s - m_new) : 0.f;
    const float corr = expf(m_run - m_new);  // 0 on the first chunk
    se[threadIdx.x] = e;
    l_run = l_run * corr + block_reduce_sum(e, red);
    m_run = m_new;
    __syncthreads();
    const int cnt = min(kThreads, L - j0);
    for (int c = threadIdx.x; c < d; c += kThreads) {
      float a = acc[c] * corr;
      for (int t = 0; t < cnt; ++t) {
        const int jj = j0 + t;
        const float* v = jj < P ? cache_row(Vcg, jj) : Vg + (size_t)(jj - P) * d;
        a = fmaf(se[t], v[c], a);
      }
      acc[c] = a;
    }
    __syncthreads();
  }
  for (int c = threadIdx.x; c < d; c += kThreads) Y[row + c] = acc[c] / l_run;
}

// The exact path with reuse for stable tokens (the LoSA page's cache reuse),
// fp32 reference mode: one CTA per (request, head, token row).  Each CTA
// evaluates its request's selection itself (the same fp64 nested sum and
// ranking as the bf16 path's selection kernel), then -- if its token is active
// (or every token is) -- its row's softmax over the cache alone (normalised
// output and natural-log normaliser into O_pre / L_pre), else reads them from
// there; then its attention over the b block tokens and the online-softmax
// merge of the two.  `active` ([n][k], or null) gets the active tokens in
// increasing order (written by the head-0 CTAs).
__global__ void __launch_bounds__(kThreads) k_reuse_f32(
    const float* __restrict__ Q, const float* __restrict__ Qprev, const float* __restrict__ Kc,
    const float* __restrict__ Vc, int P, int cap, const float* __restrict__ K,
    const float* __restrict__ V, float* __restrict__ Y, float* __restrict__ O_pre,
    float* __restrict__ L_pre, int* __restrict__ active, int k, int hq, int hkv, int b, int d,
    float scale) {
  extern __shared__ double dsm[];
  double* part = dsm;                                   // [hq * b] (selecting steps)
  float* sq = reinterpret_cast<float*>(dsm + (Qprev ? hq * b : 0));   // [d]
  float* se = sq + d;                                   // [kThreads]
  float* acc = se + kThreads;                           // [d]
  __shared__ float red[kThreads / 32];
  __shared__ double sc[64];
  __shared__ int is_act;

  const int id = blockIdx.x;
  const int i = id % b, nh = id / b;
  const int ni = nh / hq, h = nh % hq, g = h / (hq / hkv);
  const size_t row = (((size_t)ni * hq + h) * b + i) * d;
  if (threadIdx.x == 0) is_act = 1;
  if (Qprev != nullptr && k < b) {
    // per (head, token) row: groups of 8 columns, then the groups, in order
    for (int t = threadIdx.x; t < hq * b; t += kThreads) {
      const size_t rr = ((size_t)ni * hq * b + t) * d;
      double sh = 0.0;
      for (int c0 = 0; c0 < d; c0 += 8) {
        double sg = 0.0;
        for (int c = c0; c < c0 + 8 && c < d; ++c) {
          const double df = __dsub_rn((double)Q[rr + c], (double)Qprev[rr + c]);
          sg = __dadd_rn(sg, __dmul_rn(df, df));
        }
        sh = __dadd_rn(sh, sg);
      }
      part[t] = sh;
    }
    __syncthreads();
    if (threadIdx.x < b) {
      double a = 0.0;
      for (int hh = 0; hh < hq; ++hh) a = __dadd_rn(a, part[hh * b + threadIdx.x]);
      const double s = __ddiv_rn(a, (double)hq * d);
      sc[threadIdx.x] = s != s ? -INFINITY : s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int rank = 0, pos = 0;
      for (int j = 0; j < b; ++j) rank += (sc[j] > sc[i] || (sc[j] == sc[i] && j < i)) ? 1 : 0;
      is_act = rank < k;
      if (is_act && h == 0 && active != nullptr) {
        for (int t = 0; t < i; ++t) {
          int rt = 0;
          for (int j = 0; j < b; ++j) rt += (sc[j] > sc[t] || (sc[j] == sc[t] && j < t)) ? 1 : 0;
          pos += rt < k;
        }
        if (pos < k) active[(size_t)ni * k + pos] = i;
      }
    }
  } else if (Qprev != nullptr && k == 0 && threadIdx.x == 0) {
    is_act = 0;
  }
  for (int c = threadIdx.x; c < d; c += kThreads) sq[c] = Q[row + c];
  __syncthreads();
  const bool act = is_act != 0;
  const size_t lrow = ((size_t)ni * hq + h) * b + i;
  float lse_p;
  if (act) {
    const float* Kcg = Kc + ((size_t)ni * hkv + g) * cap * d;
    const float* Vcg = Vc + ((size_t)ni * hkv + g) * cap * d;
    for (int c = threadIdx.x; c < d; c += kThreads) acc[c] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    for (int j0 = 0; j0 < P; j0 += kThreads) {
      const int j = j0 + threadIdx.x;
      float s = -INFINITY;
      if (j < P) {
        float a = 0.f;
        for (int c = 0; c < d; ++c) a = fmaf(sq[c], Kcg[(size_t)j * d + c], a);
        s = a * scale;
      }
      const float m_new = fmaxf(m_run, block_reduce_max(s, red));
      const float e = j < P ? expf(s - m_new) : 0.f;
      const float corr = expf(m_run - m_new);
      se[threadIdx.x] = e;
      l_run = l_run * corr + block_reduce_sum(e, red);
      m_run = m_new;
      __syncthreads();
      const int cnt = min(kThreads, P - j0);
      for (int c = threadIdx.x; c < d; c += kThreads) {
        float a = acc[c] * corr;
        for (int t = 0; t < cnt; ++t) a = fmaf(se[t], Vcg[(size_t)(j0 + t) * d + c], a);
        acc[c] = a;
      }
      __syncthreads();
    }
    for (int c = threadIdx.x; c < d; c += kThreads) {
      acc[c] = P > 0 ? acc[c] / l_run : 0.f;
      O_pre[row + c] = acc[c];
    }
    lse_p = P > 0 ? m_run + logf(l_run) : -INFINITY;
    if (threadIdx.x == 0) L_pre[lrow] = lse_p;
  } else {
    for (int c = threadIdx.x; c < d; c += kThreads) acc[c] = O_pre[row + c];
    lse_p = L_pre[lrow];
  }
  __syncthreads();
  // the block's attention with this step's query
  const float* Kg = K + ((size_t)ni * hkv + g) * b * d;
  const float* Vg = V + ((size_t)ni * hkv + g) * b * d;
  float s = -INFINITY;
  if (threadIdx.x < b) {
    float a = 0.f;
    for (int c = 0; c < d; ++c) a = fmaf(sq[c], Kg[(size_t)threadIdx.x * d + c], a);
    s = a * scale;
  }
  const float mb = block_reduce_max(s, red);
  const float e = threadIdx.x < b ? expf(s - mb) : 0.f;
  const float lb = block_reduce_sum(e, red);
  se[threadIdx.x] = e;
  __syncthreads();
  const float lse_b = mb + logf(lb);
  const float M = fmaxf(lse_p, lse_b);
  const float wp = lse_p == -INFINITY ? 0.f : expf(lse_p - M);
  const float wb = expf(lse_b - M);
  for (int c = threadIdx.x; c < d; c += kThreads) {
    float ob = 0.f;
    for (int j = 0; j < b; ++j) ob = fmaf(se[j], Vg[(size_t)j * d + c], ob);
    ob /= lb;
    Y[row + c] = (wp * acc[c] + wb * ob) / (wp + wb);
  }
}

int finish_launch() {
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace

int launch_step_f32(const Ctx& c, const float* Q, const float* K, const float* V,
                    const float* S, const float* z, float* Y, int n, int hq, int hkv, int b,
                    int d, float scale, int shared, int fmap, const float* W) {
  const size_t smem = (size_t)(2 * b * d + 2 * d + b) * sizeof(float);
  static Prepared prepared;
  if (!prepare_kernel(c, k_step_f32, (2 * 64 * 128 + 2 * 128 + 64) * 4, prepared)) return -5;
  k_step_f32<<<n * hq, kThreads, smem, c.stream>>>(Q, K, V, S, z, Y, hq, hkv, b, d, scale,
                                                   shared, fmap, W);
  return finish_launch();
}

int launch_commit_f32(const Ctx& c, const float* K, const float* V, int units, int b, int d,
                      float* S, float* z, int fmap, const float* W, int hkv) {
  dim3 grid((d * d + kThreads - 1) / kThreads, units);
  k_state_f32<<<grid, kThreads, 0, c.stream>>>(K, V, b, d, S, z, 1, fmap, W, hkv, nullptr);
  return finish_launch();
}

int launch_prefill_f32(const Ctx& c, const float* K, const float* V, int units, int T, int d,
                       float* S, float* z, int fmap, const float* W, int hkv,
                       const int* T_lens) {
  dim3 grid((d * d + kThreads - 1) / kThreads, units);
  k_state_f32<<<grid, kThreads, 0, c.stream>>>(K, V, T, d, S, z, 0, fmap, W, hkv, T_lens);
  return finish_launch();
}

int launch_prefix_f32(const Ctx& c, const float* Q, const float* Kc, const float* Vc, int P,
                      int cap, const float* K, const float* V, float* Y, int n, int hq, int hkv,
                      int b, int d, float scale) {
  const size_t smem = (size_t)(2 * d + kThreads) * sizeof(float);
  k_prefix_f32<<<n * hq * b, kThreads, smem, c.stream>>>(Q, Kc, Vc, P, cap, K, V, Y, hq, hkv,
                                                         b, d, scale, PagedF32{});
  return finish_launch();
}

int launch_prefix_reuse_f32(const Ctx& c, const float* Q, const float* Qprev, const float* Kc,
                            const float* Vc, int P, int cap, const float* K, const float* V,
                            float* Y, float* O_pre, float* L_pre, int* active, int k, int n,
                            int hq, int hkv, int b, int d, float scale) {
  const size_t smem = (Qprev ? (size_t)hq * b * sizeof(double) : 0) +
                      (size_t)(2 * d + kThreads) * sizeof(float);
  static Prepared prepared;
  if (!prepare_kernel(c, k_reuse_f32, 8192 * 8 + (2 * 128 + kThreads) * 4, prepared)) return -5;
  k_reuse_f32<<<n * hq * b, kThreads, smem, c.stream>>>(Q, Qprev, Kc, Vc, P, cap, K, V, Y, O_pre,
                                                        L_pre, active, k, hq, hkv, b, d, scale);
  return finish_launch();
}

int launch_prefix_paged_f32(const Ctx& c, const float* Q, const float* Kpool, const float* Vpool,
                            const PagedCache& pg, const float* K, const float* V, float* Y, int n,
                            int hq, int hkv, int b, int d, float scale) {
  const size_t smem = (size_t)(2 * d + kThreads) * sizeof(float);
  const PagedF32 p{pg.table, pg.P_lens, pg.max_pages, pg.ps_log2, pg.num_pages};
  k_prefix_f32<<<n * hq * b, kThreads, smem, c.stream>>>(Q, Kpool, Vpool, 0, 0, K, V, Y, hq, hkv,
                                                         b, d, scale, p);
  return finish_launch();
}

}  // namespace bha
