// bha_prefix_softmax_reuse: the exact path with reuse of prefix attention for
// stable tokens, bf16 tensor-core path (d = 128).
//
// The method of the LoSA page (gist.science explainer of arXiv 2604.12056,
// "3. 方法论 LoSA" and "技术细节"), with a dense prefix pass over the active
// tokens instead of the page's sparse selector.  Within a denoising block,
// most tokens' queries barely change from one step to the next; their
// attention over the cached prefix is carried over from the previous step
// (its normalised output and log-normaliser, b x (d + 1) values per head),
// and only the k tokens whose queries changed most get a new prefix pass.
// Every token's attention over the active block itself is recomputed and
// merged with its prefix part by the online-softmax identity.
//
// Launch sequence of one step (each kernel with programmatic dependent
// launch, so every one waits for its predecessor before touching memory):
//   k_reuse_select       one CTA per request: the locality scores (the MSE of
//                        each token's query change over all heads, fp64, a
//                        nested sum in a fixed order so that the selection is
//                        reproducible bit for bit), the top-k active set (ties to the lower
//                        index), the active tokens' query rows packed per KV
//                        head into the workspace [units][G k][128];
//   k_prefix_bf16        (prefix-only mode) the exact path's flash kernel over
//                        the cache for the packed rows, chunk partials out;
//   k_reuse_merge        per packed row: the chunks combined by log-sum-exp,
//                        the normalised output and natural-log normaliser
//                        scattered into the token's entries of (O_pre, L_pre);
//   k_step_bf16<REUSE>   per (request, KV head, 128 rows): every row's block
//                        attention, y = a (P V) + b O_pre with the weights of
//                        the online-softmax merge.
// The first step of a block (no previous queries) or k >= b makes every token
// active: no selection, the prefix pass reads Q directly.  k = 0 makes every
// token stable: only the block pass runs.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <cstdint>

#include "bha_internal.h"
#include "bha_ptx.cuh"

namespace bha {
namespace {

constexpr int kD = 128;
constexpr int kSelThreads = 512;
constexpr int kMaxB = 64;
// per-head partial scores of one request: hq * b doubles, hq * b <= 8192
constexpr size_t kSelMaxSmem = 8192 * sizeof(double);

struct SelectArgs {
  const __nv_bfloat16* Q;      // [n][hq][b][128]
  const __nv_bfloat16* Qprev;  // [n][hq][b][128]
  __nv_bfloat16* Qact;         // [n][hkv][G k][128]: the active tokens' rows
  int* list;                   // [n][k] active tokens, increasing
  int* active_out;             // [n][k] copy for the caller, or null
  int hq, hkv, b, k;
};

__device__ __forceinline__ double bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ double bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// One CTA per request (kSelThreads threads, dynamic shared memory of hq * b
// doubles).  The score of token i is evaluated as a plain nested sum in fp64,
// each level in index order and every product and sum rounded on its own (no
// fused multiply-add): per head h and group of 8 columns, the squared query
// change summed column by column; per head the 16 group sums; over the heads
// the hq head sums; then divided by hq * 128.  Equal inputs give bit-identical
// scores wherever this is computed.  A half warp takes one (head, token) row:
// lane j of it loads columns 8j .. 8j+7 of Q and Qprev (a coalesced 256-byte
// row per half warp) and sums its group; the half warp's lane 0 then adds the
// 16 group sums in order.
constexpr int kRowsPerPass = kSelThreads / 16;   // rows in flight per pass
constexpr int kPassUnroll = 4;                   // passes whose loads issue together
__global__ void __launch_bounds__(kSelThreads) k_reuse_select(const SelectArgs a) {
  extern __shared__ double part[];   // [hq][b] per-head sums
  __shared__ double sc[kMaxB];
  __shared__ int act[kMaxB];
  __shared__ int lst[kMaxB];
  pdl_launch_dependents();
  pdl_wait();
  const int ni = blockIdx.x, tid = threadIdx.x;
  const int b = a.b, hq = a.hq;
  const int rows = hq * b;
  const int hw = tid >> 4, j = tid & 15;   // half warp = row slot, lane = column group
  const uint4* Q4 = reinterpret_cast<const uint4*>(a.Q) + static_cast<size_t>(ni) * rows * 16;
  const uint4* P4 = reinterpret_cast<const uint4*>(a.Qprev) + static_cast<size_t>(ni) * rows * 16;
  for (int r0 = 0; r0 < rows; r0 += kRowsPerPass * kPassUnroll) {
    uint4 qv[kPassUnroll], pv[kPassUnroll];
#pragma unroll
    for (int p = 0; p < kPassUnroll; ++p) {
      const int t = r0 + p * kRowsPerPass + hw;   // row t = h * b + i
      if (t < rows) {
        qv[p] = __ldg(Q4 + static_cast<size_t>(t) * 16 + j);
        pv[p] = __ldg(P4 + static_cast<size_t>(t) * 16 + j);
      }
    }
#pragma unroll
    for (int p = 0; p < kPassUnroll; ++p) {
      const int t = r0 + p * kRowsPerPass + hw;
      double g = 0.0;   // this lane's group of 8 columns
      if (t < rows) {
        const uint32_t qw[4] = {qv[p].x, qv[p].y, qv[p].z, qv[p].w};
        const uint32_t pw[4] = {pv[p].x, pv[p].y, pv[p].z, pv[p].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double d0 = __dsub_rn(bf16_lo(qw[e]), bf16_lo(pw[e]));
          g = __dadd_rn(g, __dmul_rn(d0, d0));
          const double d1 = __dsub_rn(bf16_hi(qw[e]), bf16_hi(pw[e]));
          g = __dadd_rn(g, __dmul_rn(d1, d1));
        }
      }
      // the row's 16 group sums, in order, by the half warp's lane 0
      double row = 0.0;
#pragma unroll
      for (int q = 0; q < 16; ++q) row = __dadd_rn(row, __shfl_sync(0xffffffffu, g, (tid & 16) + q));
      if (j == 0 && t < rows) part[t] = row;
    }
  }
  __syncthreads();
  if (tid < b) {
    double acc = 0.0;
    for (int h = 0; h < hq; ++h) acc = __dadd_rn(acc, part[h * b + tid]);
    const double s = __ddiv_rn(acc, static_cast<double>(hq) * kD);
    // (a NaN score -- NaN in the queries -- ranks last, so that the order
    // stays total and exactly k tokens are selected)
    sc[tid] = s != s ? -INFINITY : s;
  }
  if (tid < kMaxB) lst[tid] = 0;
  __syncthreads();
  if (tid < b) {
    // rank: tokens with a larger score, or an equal one and a lower index
    const double s = sc[tid];
    int rank = 0;
    for (int jj = 0; jj < b; ++jj) rank += (sc[jj] > s || (sc[jj] == s && jj < tid)) ? 1 : 0;
    act[tid] = rank < a.k ? 1 : 0;
  }
  __syncthreads();
  if (tid < b && act[tid]) {
    int pos = 0;
    for (int j = 0; j < tid; ++j) pos += act[j];
    if (pos < a.k) {
      lst[pos] = tid;
      a.list[static_cast<size_t>(ni) * a.k + pos] = tid;
      if (a.active_out != nullptr) a.active_out[static_cast<size_t>(ni) * a.k + pos] = tid;
    }
  }
  __syncthreads();
  // pack the active tokens' query rows: unit (ni, g), row hl * k + pos
  const int G = hq / a.hkv;
  const int per_row = kD * 2 / 16;   // 16 uint4 per row
  const int total = hq * a.k * per_row;
  for (int e = tid; e < total; e += kSelThreads) {
    const int c = e % per_row;
    const int r = e / per_row;       // h * k + pos
    const int h = r / a.k, pos = r % a.k;
    const int g = h / G, hl = h % G;
    const uint4* src = reinterpret_cast<const uint4*>(
        a.Q + ((static_cast<size_t>(ni) * hq + h) * b + lst[pos]) * kD);
    uint4* dst = reinterpret_cast<uint4*>(
        a.Qact + ((static_cast<size_t>(ni) * a.hkv + g) * (G * a.k) + hl * a.k + pos) * kD);
    dst[c] = __ldg(src + c);
  }
}

struct MergeArgs {
  const float* wsO;    // [items][128][128] chunk numerators (or null: no prefix)
  const float* wsML;   // [items][2][128] row max (log2 units), row sum
  const int* list;     // [n][k] active tokens (null: every token, packed row = token)
  float* O_pre;        // [n][hq][b][128]
  float* L_pre;        // [n][hq][b]
  int hkv, G, b, k;    // k: active tokens per request (b when all)
  int rows, mtiles, splits;   // packed rows per unit (G k), their tiles, key chunks
};

// Grid (16, units * mtiles), 256 threads: one float4 of a 128 x 128 tile per
// thread.  O_pre row = sum_s 2^{m_s - M} O_s / sum_s 2^{m_s - M} l_s, and
// L_pre = ln 2 (M + log2 sum_s 2^{m_s - M} l_s); no chunks (an empty cache):
// O_pre = 0, L_pre = -inf.
__global__ void __launch_bounds__(256) k_reuse_merge(const MergeArgs ma) {
  pdl_launch_dependents();
  pdl_wait();
  const int umt = blockIdx.y;
  const int u = umt / ma.mtiles, mt = umt % ma.mtiles;
  const int e = blockIdx.x * 256 + threadIdx.x;
  const int r = e >> 5, c4 = e & 31;
  const int prow = mt * 128 + r;   // packed row: hl * k + pos
  if (prow >= ma.rows) return;
  const int ni = u / ma.hkv, g = u % ma.hkv;
  const int hl = prow / ma.k, pos = prow % ma.k;
  const int tok = ma.list != nullptr ? __ldg(ma.list + static_cast<size_t>(ni) * ma.k + pos) : pos;
  const size_t orow = ((static_cast<size_t>(ni) * ma.hkv + g) * ma.G + hl) * ma.b + tok;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lse = -INFINITY;
  if (ma.splits > 0) {
    const size_t item0 = static_cast<size_t>(umt) * ma.splits;
    float M = -INFINITY;
    for (int s = 0; s < ma.splits; ++s) M = fmaxf(M, ma.wsML[(item0 + s) * 256 + r]);
    float den = 0.f;
    for (int s = 0; s < ma.splits; ++s) {
      const float* ml = ma.wsML + (item0 + s) * 256;
      const float w = exp2f(ml[r] - M);
      if (w == 0.f) continue;
      den = fmaf(w, ml[128 + r], den);
      const float4 o =
          reinterpret_cast<const float4*>(ma.wsO + (item0 + s) * kD * kD + r * kD)[c4];
      acc.x = fmaf(w, o.x, acc.x);
      acc.y = fmaf(w, o.y, acc.y);
      acc.z = fmaf(w, o.z, acc.z);
      acc.w = fmaf(w, o.w, acc.w);
    }
    const float inv = 1.f / den;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    lse = (M + __log2f(den)) * 0.6931471805599453f;
  }
  reinterpret_cast<float4*>(ma.O_pre + orow * kD)[c4] = acc;
  if (c4 == 0) ma.L_pre[orow] = lse;
}

constexpr size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct ReuseLayout {
  bool all_active;   // no selection: every token gets the prefix pass
  int k_eff;         // active tokens per request
  int rows;          // packed rows per unit, G * k_eff
  int splits, tiles_per;
  size_t off_list, off_qact, off_o, off_ml, total;
};

ReuseLayout reuse_layout(int n, int hq, int hkv, int b, int P, int k, bool have_prev) {
  ReuseLayout L = {};
  const int G = hq / hkv;
  const int units = n * hkv;
  L.all_active = !have_prev || k >= b;
  L.k_eff = L.all_active ? b : (k < 0 ? 0 : k);
  L.rows = G * L.k_eff;
  size_t off = 0;
  if (!L.all_active && L.k_eff > 0) {
    L.off_list = off;
    off = align256(off + static_cast<size_t>(n) * L.k_eff * sizeof(int));
    L.off_qact = off;
    off = align256(off + static_cast<size_t>(units) * L.rows * kD * 2);
  }
  if (P > 0 && L.k_eff > 0) {
    prefix_only_plan(units, L.rows, P, &L.splits, &L.tiles_per);
    const size_t items = static_cast<size_t>(units) * ((L.rows + 127) / 128) * L.splits;
    L.off_o = off;
    off = align256(off + items * kD * kD * sizeof(float));
    L.off_ml = off;
    off = align256(off + items * 256 * sizeof(float));
  }
  L.total = off;
  return L;
}

}  // namespace

size_t reuse_bf16_workspace(int n, int hq, int hkv, int b, int P, int k, int have_prev) {
  return reuse_layout(n, hq, hkv, b, P, k, have_prev != 0).total;
}

int launch_prefix_reuse_bf16(const Ctx& c, const void* Q, const void* Qprev, const void* Kc,
                             const void* Vc, int P, int cap, const void* K, const void* V,
                             void* Y, float* O_pre, float* L_pre, int* active, int k, int n,
                             int hq, int hkv, int b, float scale, void* ws, size_t ws_bytes) {
  const ReuseLayout L = reuse_layout(n, hq, hkv, b, P, k, Qprev != nullptr);
  if (L.total > ws_bytes) return -4;
  const int G = hq / hkv;
  const int units = n * hkv;
  uint8_t* w = static_cast<uint8_t*>(ws);
  const void* Qsrc = Q;
  int* list = nullptr;
  if (!L.all_active && L.k_eff > 0) {
    list = reinterpret_cast<int*>(w + L.off_list);
    SelectArgs sa;
    sa.Q = static_cast<const __nv_bfloat16*>(Q);
    sa.Qprev = static_cast<const __nv_bfloat16*>(Qprev);
    sa.Qact = reinterpret_cast<__nv_bfloat16*>(w + L.off_qact);
    sa.list = list;
    sa.active_out = active;
    sa.hq = hq;
    sa.hkv = hkv;
    sa.b = b;
    sa.k = L.k_eff;
    const size_t sel_smem = static_cast<size_t>(hq) * b * sizeof(double);
    if (sel_smem > kSelMaxSmem) return -5;   // the C ABI bounds hq * b
    static Prepared prepared;
    if (!prepare_kernel(c, k_reuse_select, static_cast<int>(kSelMaxSmem), prepared)) return -5;
    if (launch_pdl(k_reuse_select, static_cast<unsigned>(n), kSelThreads, sel_smem, c.stream,
                   sa))
      return -5;
    Qsrc = sa.Qact;
  }
  if (L.k_eff > 0) {
    float* wsO = P > 0 ? reinterpret_cast<float*>(w + L.off_o) : nullptr;
    float* wsML = P > 0 ? reinterpret_cast<float*>(w + L.off_ml) : nullptr;
    if (P > 0 && launch_prefix_partials_bf16(c, Qsrc, L.rows, Kc, Vc, P, cap, units, hkv, scale,
                                             wsO, wsML))
      return -5;
    const int mtiles = (L.rows + 127) / 128;
    MergeArgs ma;
    ma.wsO = wsO;
    ma.wsML = wsML;
    ma.list = list;
    ma.O_pre = O_pre;
    ma.L_pre = L_pre;
    ma.hkv = hkv;
    ma.G = G;
    ma.b = b;
    ma.k = L.k_eff;
    ma.rows = L.rows;
    ma.mtiles = mtiles;
    ma.splits = P > 0 ? L.splits : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kD * kD / 4 / 256, units * mtiles);
    cfg.blockDim = dim3(256);
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_reuse_merge, ma) != cudaSuccess) return -5;
    if (cudaGetLastError() != cudaSuccess) return -5;
  }
  return launch_reuse_block_bf16(c, Q, K, V, O_pre, L_pre, Y, n, hq, hkv, b, scale);
}

}  // namespace bha
