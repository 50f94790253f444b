// bha_prefix_softmax, bf16 tensor-core path (d = 128): the comparison path.
//
// Exact softmax attention of the active block's queries over the whole KV
// cache followed by the block itself -- the baseline of "Retrofitting Linear
// Attention into Diffusion Language Models" (abstract: every denoising step
// still attends to all previous blocks).  Flash-attention structure on
// tcgen05:
//   * one CTA per (request, KV head, 128-row tile of the G*b packed query
//     rows, chunk of the key sequence); keys come in 64-token tiles, cache
//     tiles first, the active block last; 113 KB of shared memory and 256
//     TMEM columns, so two CTAs share an SM and one's prologue, pipeline
//     fill and epilogue overlap the other's stream;
//   * two TMA threads stream K and V tiles through 2-stage rings (a K stage
//     is refilled once the score MMA has read it, without waiting for the V
//     stage of the same tile), an MMA thread issues S = Q K^T into one of two
//     TMEM buffers and O += P V into a TMEM accumulator, and four softmax
//     warps (thread = query row = TMEM lane) run the online softmax in
//     registers -- exponentials on the packed fp32 pipe and the SFU, the key
//     mask only in a partial tile -- rescaling O only when a row max grows by
//     more than 2^8 (the stale max is exact for the final ratio);
//   * chunks are combined by log-sum-exp in a second kernel, the way the
//     LoSA page describes merging prefix and block attention with online
//     softmax.  With one chunk the CTA normalises and stores Y itself.
// Paged variant (the summary page pairs the method with KV-cache management;
// its related work names PagedAttention): the cache of request i is its first
// P_lens[i] tokens, token t at row t % page_size of page block_table[i][t /
// page_size] of a pool [pages][hkv][page_size][128].  A 64-key tile is one
// TMA box per page (page_size < 64: 64 / page_size boxes, pages past the
// request's cache not loaded; page_size >= 64: part of one page).  A
// one-CTA planning kernel reads the lengths on the device and cuts each
// request into pieces of equal length plus a remainder, longest first (see
// k_prefix_paged_plan); each CTA takes one piece, a request of one piece
// writes Y itself, and the merge combines the pieces of the others.  Rows
// past the cache in its last tile hold stale pool data: their scores are
// masked and their V rows zeroed before P V.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>
#include <cmath>

#include "bha_internal.h"
#include "bha_ptx.cuh"

namespace bha {
namespace {

constexpr int kD = 128;
constexpr int kTK = 64;              // keys per tile
constexpr int kThreads = 256;
constexpr uint32_t kQBytes = 128 * kD * 2;      // 32 KB: 2 boxes of 64 columns
constexpr uint32_t kTileBytes = kTK * kD * 2;   // 16 KB K or V tile: 2 boxes of 8 KB
constexpr uint32_t kBox = kTK * 128;            // one 64-column box of a K / V tile
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kQBytes;                     // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;      // 2 stages
constexpr uint32_t kOffP = kOffV + 2 * kTileBytes;      // 128 rows x 64 keys bf16
constexpr uint32_t kTiles = kOffP + 128 * kTK * 2;      // 112 KB
constexpr uint32_t kCtrlBytes = 256;
constexpr uint32_t kSmem = kTiles + 1024;
constexpr uint32_t kTmemCols = 256;   // S buffers [0, 64), [64, 128); O [128, 256)
constexpr uint32_t kColO = 128;
constexpr float kRescaleLog2 = 8.f;             // rescale O when max grows > 2^8
constexpr int kMinTilesPerChunk = 16;           // 1024 keys
constexpr int kPagedTilesPerChunk = 32;         // 2048 keys

struct PrefixArgs {
  int* err;
  const int* table;  // paged: [n][max_pages] page numbers
  const int* P_lens; // paged: [n] cached tokens per request
  int max_pages;
  int ps_log2;       // paged: log2(page_size)
  int hkv;
  int Pmax;          // paged: max_pages * page_size
  const int* hdr;    // paged plan: [0] tiles per piece, [1] pieces (null: fixed chunks)
  const int4* work;  // paged plan: (unit row, piece, first tile, tiles), longest first
  float* wsO;        // [items][128][128] fp32 partial numerators (splits > 1)
  float* wsML;       // [items][2][128] row max (log2 units) and row sum
  int rows;          // G * b
  int mtiles;
  int P;             // cached tokens
  int b;             // active-block tokens
  int ncache_tiles;  // ceil(P / 128)
  int splits;
  int tiles_per;
  float sl2;         // scale * log2(e)
  int prefix_only;   // reuse path: cache tiles only (no block tile), partials always
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

template <bool PAGED>
__global__ void __launch_bounds__(kThreads, 2)
    k_prefix_bf16(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKc,
                  const __grid_constant__ CUtensorMap tmVc, const __grid_constant__ CUtensorMap tmKa,
                  const __grid_constant__ CUtensorMap tmVa, const __grid_constant__ CUtensorMap tmY,
                  const __grid_constant__ CUtensorMap tmO, const PrefixArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x;
  // (unit row, chunk) of this CTA; the paged plan's work list replaces the
  // fixed chunking once the plan is visible (after pdl_wait)
  int sp = item % a.splits;
  int umt = item / a.splits;
  int tile0 = sp * a.tiles_per;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t ctrl = (base - raw >= kCtrlBytes) ? raw : base + kTiles;
  uint8_t* ctrl_ptr = smem_raw + (ctrl - raw);
  const uint32_t bar_q = ctrl, bar_kf = ctrl + 8, bar_ke = ctrl + 24, bar_vf = ctrl + 40,
                 bar_ve = ctrl + 56, bar_sf = ctrl + 72, bar_pf = ctrl + 88, bar_pv = ctrl + 96;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl_ptr + 104);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl_ptr + 108);

  // softmax warps with query rows in this tile (a ragged last tile, the reuse
  // path's packed active rows); with a contiguous cache the others take no
  // part in P's barrier at all
  const int mt0 = (item / a.splits) % a.mtiles;
  const int live_warps = PAGED ? 4 : min(4, max(1, (a.rows - mt0 * 128 + 31) / 32));
  if (warp == 0) {
    if (lane == 0) {
      mbar_init(bar_q, 1);
      for (int s = 0; s < 2; ++s) {
        mbar_init(bar_kf + 8 * s, 1);
        mbar_init(bar_ke + 8 * s, 1);
        mbar_init(bar_vf + 8 * s, 1);
        mbar_init(bar_ve + 8 * s, 1);
        mbar_init(bar_sf + 8 * s, 1);
      }
      mbar_init(bar_pf, 32 * live_warps);
      mbar_init(bar_pv, 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_o = tmem + kColO;
  pdl_wait();

  int nt_plan = a.tiles_per;
  bool planned = true;
  if (PAGED && a.work != nullptr) {
    planned = item < __ldcg(a.hdr + 1);
    if (planned) {
      const int4 w = __ldcg(a.work + item);
      umt = w.x;
      sp = w.y;
      tile0 = w.z;
      nt_plan = w.w;
    } else {
      umt = 0;
      sp = 0;
      tile0 = 0;
    }
  }
  const int u = umt / a.mtiles, mt = umt % a.mtiles;
  // this request's cache length (per request when paged), tiles of this chunk
  const int nreq = u / a.hkv, g = u % a.hkv;
  const int P = PAGED ? min(max(__ldg(a.P_lens + nreq), 0), a.Pmax) : a.P;
  const int ncache_tiles = PAGED ? (P + kTK - 1) / kTK : a.ncache_tiles;
  const int key_tiles = ncache_tiles + (a.prefix_only ? 0 : 1);
  const int nt = planned ? max(0, min(nt_plan, key_tiles - tile0)) : 0;
  // false for a chunk past a paged request's cache, or past the plan's pieces
  const bool live = nt > 0;
  // pieces of this unit row: one writes Y directly, more write partials
  int npieces = a.splits;
  if (PAGED && a.work != nullptr) {
    const int L = __ldcg(a.hdr);
    npieces = min(a.splits, (ncache_tiles + 1 + L - 1) / L);
  }
  // the reuse path's prefix pass hands every chunk to its merge as a partial
  const bool direct = npieces == 1 && !a.prefix_only;
  const int slot = umt * a.splits + sp;   // partial numerator slot

  // loads one K or V tile of the cache (through the page table) or of the block
  auto load_tile = [&](const CUtensorMap* mc, const CUtensorMap* ma, uint32_t dst, uint32_t bar,
                       int gi) {
    if (gi >= ncache_tiles) {
      mbar_arrive_expect_tx(bar, kTileBytes);
      tma_load_3d(dst, ma, bar, 0, 0, u);
      tma_load_3d(dst + kBox, ma, bar, 64, 0, u);
    } else if (!PAGED) {
      mbar_arrive_expect_tx(bar, kTileBytes);
      tma_load_3d(dst, mc, bar, 0, gi * kTK, u);
      tma_load_3d(dst + kBox, mc, bar, 64, gi * kTK, u);
    } else {
      const int t0 = gi * kTK;
      const int* trow = a.table + static_cast<size_t>(nreq) * a.max_pages;
      if (a.ps_log2 >= 6) {
        // part of one page
        const int pg = __ldg(trow + (t0 >> a.ps_log2));
        const int row = t0 & ((1 << a.ps_log2) - 1);
        mbar_arrive_expect_tx(bar, kTileBytes);
        tma_load_3d(dst, mc, bar, 0, row, pg * a.hkv + g);
        tma_load_3d(dst + kBox, mc, bar, 64, row, pg * a.hkv + g);
      } else {
        // 64 / page_size pages; only those holding cached tokens
        const int ps = 1 << a.ps_log2;
        const int npg = min(kTK >> a.ps_log2, (P - t0 + ps - 1) >> a.ps_log2);
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(npg) * ps * 256);
        for (int j = 0; j < npg; ++j) {
          const int pg = __ldg(trow + (t0 >> a.ps_log2) + j);
          tma_load_3d(dst + j * ps * 128, mc, bar, 0, 0, pg * a.hkv + g);
          tma_load_3d(dst + kBox + j * ps * 128, mc, bar, 64, 0, pg * a.hkv + g);
        }
      }
    }
  };
  if (tid == 0 && live) {
    // ---------------- TMA producer of Q and the K ring: a K stage is free
    // once the score MMA has read it, well before P V frees the V stage of
    // the same tile, so the two rings are refilled by separate threads
    const int row0 = mt * 128;
    mbar_arrive_expect_tx(bar_q, kQBytes);
    tma_load_3d(base + kOffQ, &tmQ, bar_q, 0, row0, u);
    tma_load_3d(base + kOffQ + 16384, &tmQ, bar_q, 64, row0, u);
    for (int i = 0; i < nt; ++i) {
      const int st = i & 1;
      if (i >= 2 && !mbar_wait(bar_ke + 8 * st, ((i >> 1) - 1) & 1, a.err, abort_flag)) break;
      load_tile(&tmKc, &tmKa, base + kOffK + st * kTileBytes, bar_kf + 8 * st, tile0 + i);
    }
  } else if (tid == 64 && live) {
    // ---------------- TMA producer of the V ring
    for (int i = 0; i < nt; ++i) {
      const int st = i & 1;
      if (i >= 2 && !mbar_wait(bar_ve + 8 * st, ((i >> 1) - 1) & 1, a.err, abort_flag)) break;
      load_tile(&tmVc, &tmVa, base + kOffV + st * kTileBytes, bar_vf + 8 * st, tile0 + i);
    }
  } else if (tid == 32 && live) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc_s = make_idesc_bf16(128, kTK, 0, 0);   // Q K^T, both K-major
    constexpr uint32_t idesc_o = make_idesc_bf16(128, kD, 0, 1);    // P V, V MN-major
    bool ok = mbar_wait(bar_q, 0, a.err, abort_flag);
    auto issue_s = [&](int i) -> bool {
      const int st = i & 1;
      if (!mbar_wait(bar_kf + 8 * st, (i >> 1) & 1, a.err, abort_flag)) return false;
      tc_fence_after();
      const uint32_t kb = base + kOffK + st * kTileBytes;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t da =
            make_sdesc(base + kOffQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128);
        const uint64_t db = make_sdesc(kb + (ks >> 2) * kBox + (ks & 3) * 32, 16, 1024,
                                       kLayoutSW128);
        mma_bf16_ss(tmem + st * kTK, da, db, idesc_s, ks > 0 ? 1u : 0u);
      }
      mma_commit(bar_sf + 8 * st);
      mma_commit(bar_ke + 8 * st);
      return true;
    };
    if (ok && nt > 0) ok = issue_s(0);
    for (int i = 0; i < nt && ok; ++i) {
      if (i + 1 < nt) ok = issue_s(i + 1);
      if (!ok) break;
      const int st = i & 1;
      ok = mbar_wait(bar_pf, i & 1, a.err, abort_flag) &&
           mbar_wait(bar_vf + 8 * st, (i >> 1) & 1, a.err, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t vb = base + kOffV + st * kTileBytes;
#pragma unroll
      for (int ks = 0; ks < kTK / 16; ++ks) {
        // P: 128 rows of 64 keys (K-major, SW128)
        const uint64_t da = make_sdesc(base + kOffP + ks * 32, 16, 1024, kLayoutSW128);
        // V tile: [keys][d] as 2 boxes of 64 d-columns; keys are the K dim
        const uint64_t db = make_sdesc(vb + ks * 2048, kBox, 1024, kLayoutSW128);
        mma_bf16_ss(t_o, da, db, idesc_o, (i | ks) ? 1u : 0u);
      }
      mma_commit(bar_ve + 8 * st);
      mma_commit(bar_pv);
    }
  }

  // ---------------- softmax warps: thread = query row = TMEM lane
  float mx = -INFINITY, l = 0.f;
  const int r = (warp & 3) * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  bool ok = true;
  // a warp whose 32 query rows are all past the tile's valid rows (a ragged
  // last query tile, the reuse path's packed active rows) computes no
  // softmax; paged, it keeps the barrier protocol and its share of clearing
  // the V rows past the cache, which every output row's P V reads
  const bool rows_live = mt * 128 + (warp & 3) * 32 < a.rows;
  if (warp >= 4 && live && !rows_live && PAGED) {
    for (int i = 0; i < nt; ++i) {
      const int st = i & 1;
      const int gi = tile0 + i;
      if (i > 0) {
        ok = warp_all(ok && mbar_wait(bar_pv, (i - 1) & 1, a.err, abort_flag));
        if (!ok) break;
      }
      if (PAGED && gi < ncache_tiles && P - gi * kTK < kTK) {
        ok = warp_all(ok && mbar_wait(bar_vf + 8 * st, (i >> 1) & 1, a.err, abort_flag));
        if (!ok) break;
        if (r >= P - gi * kTK && r < kTK) {
          const uint32_t vrow = base + kOffV + st * kTileBytes + r * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            st_shared_v4(vrow + q * 16, 0u, 0u, 0u, 0u);
            st_shared_v4(vrow + kBox + q * 16, 0u, 0u, 0u, 0u);
          }
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(bar_pf);
    }
    if (ok && nt > 0) ok = warp_all(mbar_wait(bar_pv, (nt - 1) & 1, a.err, abort_flag));
  } else if (warp >= 4 && live && rows_live) {
    for (int i = 0; i < nt; ++i) {
      const int st = i & 1;
      const int gi = tile0 + i;
      const int valid = gi < ncache_tiles ? min(kTK, P - gi * kTK) : a.b;
      ok = warp_all(ok && mbar_wait(bar_sf + 8 * st, (i >> 1) & 1, a.err, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float s[kTK];
#pragma unroll
      for (int c = 0; c < kTK; c += 32) {
        float t[32];
        tmem_ld32_sync(tmem + st * kTK + lane_base + c, t);
#pragma unroll
        for (int q = 0; q < 32; ++q) s[c + q] = t[q];
      }
      // keys past the cache (the last cache tile) or the block (its tile)
      if (valid < kTK) {
#pragma unroll
        for (int j = 0; j < kTK; ++j)
          if (j >= valid) s[j] = -INFINITY;
      }
      float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int j = 4; j < kTK; j += 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], s[j + q]);
      }
      const float tmax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      float corr = 1.f;
      bool resc = false;
      if (mx == -INFINITY) {
        mx = tmax;
      } else if ((tmax - mx) * a.sl2 > kRescaleLog2) {
        corr = exp2f((mx - tmax) * a.sl2);
        mx = tmax;
        resc = true;
      }
      // p = 2^{(s - mx) scale log2 e}, as s * (scale log2 e) - mx (scale log2 e)
      const float2 sl = make_float2(a.sl2, a.sl2);
      const float2 nb = make_float2(-mx * a.sl2, -mx * a.sl2);
      float2 ls4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int j = 0; j < kTK; j += 2) {
        float2 x = fma2(make_float2(s[j], s[j + 1]), sl, nb);
        x.x = ex2_sfu(x.x);
        x.y = ex2_sfu(x.y);
        s[j] = x.x;
        s[j + 1] = x.y;
        ls4[(j >> 1) & 3] = add2(ls4[(j >> 1) & 3], x);
      }
      const float2 ls2 = add2(add2(ls4[0], ls4[1]), add2(ls4[2], ls4[3]));
      l = l * corr + (ls2.x + ls2.y);
      // P and O are free once P V of the previous tile has completed
      if (i > 0) {
        ok = warp_all(mbar_wait(bar_pv, (i - 1) & 1, a.err, abort_flag));
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int c = 0; c < kD; c += 32) {
            float o[32];
            tmem_ld32_sync(t_o + lane_base + c, o);
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] *= corr;
            tmem_st32_sync(t_o + lane_base + c, o);
          }
        }
      }
      if (PAGED && gi < ncache_tiles && valid < kTK) {
        // rows past the cache hold stale pool data (or none was loaded):
        // zero them in V so that P (0 there) times V stays finite
        ok = warp_all(mbar_wait(bar_vf + 8 * st, (i >> 1) & 1, a.err, abort_flag));
        if (!ok) break;
        if (r >= valid && r < kTK) {
          const uint32_t vrow = base + kOffV + st * kTileBytes + r * 128;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            st_shared_v4(vrow + q * 16, 0u, 0u, 0u, 0u);
            st_shared_v4(vrow + kBox + q * 16, 0u, 0u, 0u, 0u);
          }
        }
      }
      {
        const uint32_t prow = base + kOffP + r * 128;
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float* e = s + jj * 8;
          st_shared_v4(prow + ((jj ^ (r & 7)) << 4), pack_bf16x2(e[0], e[1]),
                       pack_bf16x2(e[2], e[3]), pack_bf16x2(e[4], e[5]), pack_bf16x2(e[6], e[7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_pf);
    }
    // final accumulator
    if (ok && nt > 0) ok = warp_all(mbar_wait(bar_pv, (nt - 1) & 1, a.err, abort_flag));
    tc_fence_after();
    if (ok) {
      if (direct) {
        const float inv = 1.f / l;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float o[32];
          tmem_ld32_sync(t_o + lane_base + cc * 32, o);
          const uint32_t row = base + kOffQ + (cc >> 1) * 16384 + r * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int j = (cc & 1) * 4 + q;
            const float* e = o + 8 * q;
            st_shared_v4(row + ((j ^ (r & 7)) << 4), pack_bf16x2(e[0] * inv, e[1] * inv),
                         pack_bf16x2(e[2] * inv, e[3] * inv), pack_bf16x2(e[4] * inv, e[5] * inv),
                         pack_bf16x2(e[6] * inv, e[7] * inv));
          }
        }
      } else {
#pragma unroll 1
        for (int bx = 0; bx < 4; ++bx) {
          float o[32];
          tmem_ld32_sync(t_o + lane_base + bx * 32, o);
          const uint32_t row = base + kOffK + bx * 16384 + r * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_f4(row + ((j ^ (r & 7)) << 4),
                         make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]));
        }
        float* ml = a.wsML + static_cast<size_t>(slot) * 256;
        ml[r] = mx * a.sl2;
        ml[128 + r] = l;
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && live && !*abort_flag) {
    if (direct) {
      tma_store_3d(&tmY, base + kOffQ, 0, mt * 128, u);
      tma_store_3d(&tmY, base + kOffQ + 16384, 64, mt * 128, u);
    } else {
#pragma unroll
      for (int bx = 0; bx < 4; ++bx) tma_store_3d(&tmO, base + kOffK + bx * 16384, 32 * bx, 0, slot);
    }
    bulk_commit_group();
    bulk_wait_group_read0();
  }
  __syncwarp();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// y[r][c] = sum_s 2^{m_s - M} O_s[r][c] / sum_s 2^{m_s - M} l_s,  M = max_s m_s,
// over the chunks the request has (all of them, unless paged).
struct MergeArgs {
  int rows, mtiles, splits;
  const int* P_lens;   // paged: [n] cached tokens, else null
  int hkv, Pmax, tiles_per;
  const int* hdr;      // paged plan ([0] = tiles per piece), or null
};

__global__ void __launch_bounds__(256) k_prefix_merge(const float* __restrict__ wsO,
                                                      const float* __restrict__ wsML,
                                                      __nv_bfloat16* __restrict__ Y,
                                                      const MergeArgs ma) {
  pdl_launch_dependents();
  pdl_wait();
  const int rows = ma.rows, mtiles = ma.mtiles;
  const int umt = blockIdx.y;
  const int u = umt / mtiles, mt = umt % mtiles;
  int splits = ma.splits;
  if (ma.P_lens != nullptr) {
    const int P = min(max(__ldg(ma.P_lens + u / ma.hkv), 0), ma.Pmax);
    const int per = ma.hdr != nullptr ? __ldcg(ma.hdr) : ma.tiles_per;
    splits = min(splits, ((P + kTK - 1) / kTK + 1 + per - 1) / per);
    if (ma.hdr != nullptr && splits == 1) return;   // the piece wrote Y itself
  }
  const int e = blockIdx.x * 256 + threadIdx.x;      // float4 index in the 128 x 128 tile
  const int r = e >> 5, c4 = e & 31;
  const int grow = mt * 128 + r;
  if (grow >= rows) return;
  const size_t item0 = static_cast<size_t>(umt) * ma.splits;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, wsML[(item0 + s) * 256 + r]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  // four chunks' loads in flight at a time, then one by one; a chunk of no
  // weight (a row underflow) contributes nothing, whatever its partial holds
  auto add = [&](float w, float l, float4 o) {
    if (w == 0.f) return;
    den = fmaf(w, l, den);
    acc.x = fmaf(w, o.x, acc.x);
    acc.y = fmaf(w, o.y, acc.y);
    acc.z = fmaf(w, o.z, acc.z);
    acc.w = fmaf(w, o.w, acc.w);
  };
  int s = 0;
  for (; s + 4 <= splits; s += 4) {
    float w[4], l[4];
    float4 o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float* ml = wsML + (item0 + s + j) * 256;
      w[j] = exp2f(ml[r] - M);
      l[j] = ml[128 + r];
      o[j] = reinterpret_cast<const float4*>(wsO + (item0 + s + j) * kD * kD + r * kD)[c4];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) add(w[j], l[j], o[j]);
  }
  for (; s < splits; ++s) {
    const float* ml = wsML + (item0 + s) * 256;
    const float w = exp2f(ml[r] - M);
    if (w == 0.f) continue;
    add(w, ml[128 + r], reinterpret_cast<const float4*>(wsO + (item0 + s) * kD * kD + r * kD)[c4]);
  }
  const float inv = 1.f / den;
  __nv_bfloat162* out = reinterpret_cast<__nv_bfloat162*>(
      Y + (static_cast<size_t>(u) * rows + grow) * kD + c4 * 4);
  out[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  out[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
}

// Paged plan, one CTA ahead of the exact-path kernel, from the lengths in
// device memory (so the launch sequence stays graph-capturable): each
// request's key tiles (its cache tiles plus the block's) are cut into pieces
// of exactly L tiles and one remainder, L = max(kPagedTilesPerChunk, total
// tiles / CTA slots), and the pieces are listed longest first (64 length
// buckets): the block scheduler hands CTAs out in index order, so the
// remainders fill in behind the full pieces.  Only requests longer than L are
// split, which keeps the chunk partials (written, then read back by the
// merge) few.  Measured on lengths uniform in [1, 16384]: 0.203 ms at batch 64
// against 0.221 ms with each request split evenly into pieces for two waves
// (pieces of similar but unequal length pack worse) and 0.229 ms with fixed
// 32-tile chunks over the longest cache; 0.804 ms against 0.818 and 0.89 ms
// at batch 256.  L >= total / (waves * slots), or L is the minimum and above
// it, so there are at most waves * slots + (unit rows) pieces: the launch
// needs no more CTAs.  Every unit row of a request (KV heads x query tiles)
// gets the same pieces.
struct PlanArgs {
  const int* P_lens;  // [n] cached tokens
  int n;
  int rows_per_req;   // hkv * mtiles
  int Pmax;
  int maxpieces;      // pieces per unit row at most (the workspace's slots)
  int slots;          // resident CTAs of the exact-path kernel on the device
  int cap;            // CTAs of the exact-path launch (>= pieces by construction)
  int* err;           // device error word
  int* hdr;           // out: [0] = L, [1] = pieces (work items)
  int4* work;         // out: (unit row, piece, first tile, tiles)
};
constexpr int kPlanThreads = 1024;
constexpr int kPlanWaves = 1;       // pieces for about this many waves of CTAs
constexpr int kPlanBuckets = 64;

__device__ __forceinline__ int plan_bucket(int nt, int L) {
  const long long k = static_cast<long long>(L - nt) * kPlanBuckets / L;
  return static_cast<int>(k < 0 ? 0 : (k >= kPlanBuckets ? kPlanBuckets - 1 : k));
}

__global__ void __launch_bounds__(kPlanThreads) k_prefix_paged_plan(const PlanArgs pa) {
  __shared__ unsigned long long tsum;
  __shared__ int hist[kPlanBuckets];
  __shared__ int offs[kPlanBuckets];
  __shared__ int Ls;
  const int tid = threadIdx.x;
  if (tid == 0) tsum = 0ull;
  if (tid < kPlanBuckets) hist[tid] = 0;
  pdl_launch_dependents();
  pdl_wait();
  __syncthreads();
  auto tiles_of = [&](int i) {
    const int P = min(max(__ldg(pa.P_lens + i), 0), pa.Pmax);
    return (P + kTK - 1) / kTK + 1;
  };
  unsigned long long part = 0ull;
  for (int i = tid; i < pa.n; i += kPlanThreads) part += static_cast<unsigned long long>(tiles_of(i));
  atomicAdd(&tsum, part);
  __syncthreads();
  if (tid == 0) {
    const unsigned long long total = tsum * static_cast<unsigned long long>(pa.rows_per_req);
    const unsigned long long want = static_cast<unsigned long long>(pa.slots) * kPlanWaves;
    unsigned long long per = (total + want - 1) / want;
    if (per < static_cast<unsigned long long>(kPagedTilesPerChunk)) per = kPagedTilesPerChunk;
    if (per > (1ull << 30)) per = 1ull << 30;
    Ls = static_cast<int>(per);
  }
  __syncthreads();
  const int L = Ls;
  for (int i = tid; i < pa.n; i += kPlanThreads) {
    const int t = tiles_of(i);
    const int np = min(pa.maxpieces, (t + L - 1) / L);
    const int len = max(L, (t + np - 1) / np);   // L unless np was capped
    for (int j = 0; j < np; ++j)
      atomicAdd(&hist[plan_bucket(min(len, t - j * len), L)], pa.rows_per_req);
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int k = 0; k < kPlanBuckets; ++k) {
      offs[k] = acc;
      acc += hist[k];
    }
    pa.hdr[0] = L;
    pa.hdr[1] = min(acc, pa.cap);
    if (acc > pa.cap) atomicExch(pa.err, kDevErrDevice);   // cannot happen (see above)
  }
  __syncthreads();
  for (int i = tid; i < pa.n; i += kPlanThreads) {
    const int t = tiles_of(i);
    const int np = min(pa.maxpieces, (t + L - 1) / L);
    const int len = max(L, (t + np - 1) / np);   // L unless np was capped
    for (int j = 0; j < np; ++j) {
      const int nt = min(len, t - j * len);
      const int pos = atomicAdd(&offs[plan_bucket(nt, L)], pa.rows_per_req);
      for (int k = 0; k < pa.rows_per_req; ++k)
        pa.work[pos + k] = make_int4(i * pa.rows_per_req + k, j, j * len, nt);
    }
  }
}

// Paged: at most one piece per kPagedTilesPerChunk tiles of the longest cache
// (the workspace's partial slots); the plan above decides the pieces.
void prefix_plan_paged(int P, int* splits, int* tiles_per) {
  const int ntot = (P + kTK - 1) / kTK + 1;
  const int tp = ntot < kPagedTilesPerChunk ? ntot : kPagedTilesPerChunk;
  *splits = (ntot + tp - 1) / tp;
  *tiles_per = tp;
}

// Chunking of the keys: the chunk count s (chunks of at least 16 tiles)
// that maximises the expected use of the machine -- the filled fraction of
// the last wave of CTAs (two per SM on 148 SMs) times the share of traffic
// that is not chunk partials (64 KB numerator + row statistics, written and
// read back, per chunk).  Depends only on the shapes, so the workspace query
// and the launch agree.
void prefix_plan(int units, int mtiles, int P, int* splits, int* tiles_per,
                 int block_tiles = 1) {
  constexpr double kSlots = 296.0;
  const int ntot = (P + kTK - 1) / kTK + block_tiles;
  const int items = units * mtiles;
  const int cap = (ntot + kMinTilesPerChunk - 1) / kMinTilesPerChunk;
  const double unit_bytes = static_cast<double>(ntot) * kTK * kD * 2 * 2;   // K and V
  int best = 1;
  double best_score = -1.0;
  for (int s = 1; s <= cap && s <= 64; ++s) {
    const double waves = items * s / kSlots;
    const double fill = waves / std::ceil(waves);
    const double partial = s > 1 ? s * 2.0 * (kD * kD + 256) * 4 / unit_bytes : 0.0;
    const double score = fill * (1.0 - partial);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = s;
    }
  }
  const int tp = (ntot + best - 1) / best;
  *splits = (ntot + tp - 1) / tp;
  *tiles_per = tp;
}

bool bf16_rows_tmap(CUtensorMap* m, const void* X, uint64_t rows, uint64_t row_stride_elems,
                    uint64_t units, uint32_t box_rows) {
  const uint64_t dims[3] = {(uint64_t)kD, rows, units};
  const uint64_t strides[2] = {kD * 2ull, row_stride_elems * kD * 2ull};
  const uint32_t box[3] = {64, box_rows, 1};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, X, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

namespace {

constexpr size_t kPlanHdrBytes = 256;

size_t workspace_for(int n, int hq, int hkv, int b, int P, bool paged) {
  const int units = n * hkv;
  const int rows = (hq / hkv) * b;
  const int mtiles = (rows + 127) / 128;
  int splits, tp;
  if (paged)
    prefix_plan_paged(P, &splits, &tp);
  else
    prefix_plan(units, mtiles, P, &splits, &tp);
  if (splits <= 1) return 0;
  const size_t items = static_cast<size_t>(units) * mtiles * splits;
  size_t bytes = items * (kD * kD + 256) * sizeof(float);
  if (paged) bytes += kPlanHdrBytes + items * sizeof(int4);   // the plan
  return bytes;
}

}  // namespace

size_t prefix_bf16_workspace(int n, int hq, int hkv, int b, int P) {
  return workspace_for(n, hq, hkv, b, P, false);
}

size_t prefix_paged_bf16_workspace(int n, int hq, int hkv, int b, int Pmax) {
  return workspace_for(n, hq, hkv, b, Pmax, true);
}

namespace {

// Shared by the contiguous and the paged launch; P is the cache length (the
// longest possible one when paged).
int launch_prefix_impl(const Ctx& c, const void* Q, const void* Kc, const void* Vc, int P, int cap,
                       const PagedCache* pg, const void* K, const void* V, void* Y, int n, int hq,
                       int hkv, int b, float scale, void* ws, size_t ws_bytes) {
  const int units = n * hkv;
  const int rows = (hq / hkv) * b;
  const int mtiles = (rows + 127) / 128;
  int splits, tp;
  if (pg != nullptr)
    prefix_plan_paged(P, &splits, &tp);
  else
    prefix_plan(units, mtiles, P, &splits, &tp);
  const size_t need = workspace_for(n, hq, hkv, b, P, pg != nullptr);
  if (need > ws_bytes) return -4;
  const size_t items = static_cast<size_t>(units) * mtiles * splits;
  float* wsO = splits > 1 ? static_cast<float*>(ws) : nullptr;
  float* wsML = splits > 1 ? wsO + items * kD * kD : nullptr;
  // paged with several pieces possible: the device-side plan follows the partials
  const bool planned = pg != nullptr && splits > 1;
  int* hdr = planned ? reinterpret_cast<int*>(wsML + items * 256) : nullptr;
  // CTAs of the paged launch: every piece, never more than the slots
  const size_t plan_grid =
      planned ? std::min(items, static_cast<size_t>(kPlanWaves) * 2 * c.sm_count +
                                    static_cast<size_t>(units) * mtiles)
              : items;
  int4* work = planned ? reinterpret_cast<int4*>(reinterpret_cast<uint8_t*>(hdr) + kPlanHdrBytes)
                       : nullptr;

  CUtensorMap tq, ty, tkc, tvc, tka, tva, to;
  bool ok = bf16_rows_tmap(&tq, Q, rows, rows, units, 128) &&
            bf16_rows_tmap(&ty, Y, rows, rows, units, 128) &&
            bf16_rows_tmap(&tka, K, b, b, units, kTK) && bf16_rows_tmap(&tva, V, b, b, units, kTK);
  if (pg != nullptr) {
    // the pool as (128 columns, page rows, page * hkv + kv head)
    const int ps = 1 << pg->ps_log2;
    const uint32_t box_rows = ps < kTK ? ps : kTK;
    const uint64_t units_pool = static_cast<uint64_t>(pg->num_pages) * hkv;
    ok = ok && bf16_rows_tmap(&tkc, Kc, ps, ps, units_pool, box_rows) &&
         bf16_rows_tmap(&tvc, Vc, ps, ps, units_pool, box_rows);
  } else if (P > 0) {
    ok = ok && bf16_rows_tmap(&tkc, Kc, P, cap, units, kTK) &&
         bf16_rows_tmap(&tvc, Vc, P, cap, units, kTK);
  } else {
    tkc = tka;   // never read: there are no cache tiles
    tvc = tva;
  }
  if (splits > 1) {
    const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)kD, items};
    const uint64_t strides[2] = {kD * 4ull, (uint64_t)kD * kD * 4ull};
    const uint32_t box[3] = {32, 128, 1};
    ok = ok && encode_tmap(&to, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, wsO, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    to = ty;     // never used with one chunk
  }
  if (!ok) return -5;
  PrefixArgs a;
  a.err = c.dev_err;
  a.table = pg ? pg->table : nullptr;
  a.P_lens = pg ? pg->P_lens : nullptr;
  a.max_pages = pg ? pg->max_pages : 0;
  a.ps_log2 = pg ? pg->ps_log2 : 0;
  a.hkv = hkv;
  a.Pmax = P;
  a.hdr = hdr;
  a.work = work;
  a.wsO = wsO;
  a.wsML = wsML;
  a.rows = rows;
  a.mtiles = mtiles;
  a.P = P;
  a.b = b;
  a.ncache_tiles = (P + kTK - 1) / kTK;
  a.splits = splits;
  a.tiles_per = tp;
  a.sl2 = scale * 1.4426950408889634f;
  a.prefix_only = 0;
  int rc;
  if (planned) {
    const PlanArgs pa{pg->P_lens, n, hkv * mtiles, P, splits, 2 * c.sm_count,
                      static_cast<int>(plan_grid), c.dev_err, hdr, work};
    if (launch_pdl(k_prefix_paged_plan, 1u, kPlanThreads, 0u, c.stream, pa)) return -5;
  }
  if (pg != nullptr) {
    static Prepared prepared;
    if (!prepare_kernel(c, k_prefix_bf16<true>, (int)kSmem, prepared)) return -5;
    rc = launch_pdl(k_prefix_bf16<true>, (unsigned)plan_grid, kThreads, kSmem, c.stream, tq, tkc, tvc,
                    tka, tva, ty, to, a);
  } else {
    static Prepared prepared;
    if (!prepare_kernel(c, k_prefix_bf16<false>, (int)kSmem, prepared)) return -5;
    rc = launch_pdl(k_prefix_bf16<false>, (unsigned)items, kThreads, kSmem, c.stream, tq, tkc,
                    tvc, tka, tva, ty, to, a);
  }
  if (rc) return -5;
  if (splits > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kD * kD / 4 / 256, units * mtiles);
    cfg.blockDim = dim3(256);
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const MergeArgs ma{rows, mtiles, splits, pg ? pg->P_lens : nullptr, hkv, P, tp, hdr};
    if (cudaLaunchKernelEx(&cfg, k_prefix_merge, static_cast<const float*>(wsO),
                           static_cast<const float*>(wsML), static_cast<__nv_bfloat16*>(Y),
                           ma) != cudaSuccess)
      return -5;
    if (cudaGetLastError() != cudaSuccess) return -5;
  }
  return 0;
}

}  // namespace

// The reuse path's prefix pass: `rows` packed query rows per unit, the cache
// only (no block tile), every chunk a partial (wsO, wsML), P > 0.
void prefix_only_plan(int units, int rows, int P, int* splits, int* tiles_per) {
  prefix_plan(units, (rows + 127) / 128, P, splits, tiles_per, 0);
}

int launch_prefix_partials_bf16(const Ctx& c, const void* Q, int rows, const void* Kc,
                                const void* Vc, int P, int cap, int units, int hkv, float scale,
                                float* wsO, float* wsML) {
  const int mtiles = (rows + 127) / 128;
  int splits, tp;
  prefix_only_plan(units, rows, P, &splits, &tp);
  const size_t items = static_cast<size_t>(units) * mtiles * splits;
  CUtensorMap tq, tkc, tvc, to;
  bool ok = bf16_rows_tmap(&tq, Q, rows, rows, units, 128) &&
            bf16_rows_tmap(&tkc, Kc, P, cap, units, kTK) &&
            bf16_rows_tmap(&tvc, Vc, P, cap, units, kTK);
  const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)kD, items};
  const uint64_t strides[2] = {kD * 4ull, (uint64_t)kD * kD * 4ull};
  const uint32_t box[3] = {32, 128, 1};
  ok = ok && encode_tmap(&to, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, wsO, dims, strides, box,
                         CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return -5;
  PrefixArgs a = {};
  a.err = c.dev_err;
  a.hkv = hkv;
  a.Pmax = P;
  a.wsO = wsO;
  a.wsML = wsML;
  a.rows = rows;
  a.mtiles = mtiles;
  a.P = P;
  a.b = 0;
  a.ncache_tiles = (P + kTK - 1) / kTK;
  a.splits = splits;
  a.tiles_per = tp;
  a.sl2 = scale * 1.4426950408889634f;
  a.prefix_only = 1;
  static Prepared prepared;
  if (!prepare_kernel(c, k_prefix_bf16<false>, (int)kSmem, prepared)) return -5;
  // the block maps are never read (no block tile) and Y is never written
  return launch_pdl(k_prefix_bf16<false>, (unsigned)items, kThreads, kSmem, c.stream, tq, tkc,
                    tvc, tkc, tvc, tq, to, a)
             ? -5
             : 0;
}

int launch_prefix_bf16(const Ctx& c, const void* Q, const void* Kc, const void* Vc, int P,
                       int cap, const void* K, const void* V, void* Y, int n, int hq, int hkv,
                       int b, float scale, void* ws, size_t ws_bytes) {
  return launch_prefix_impl(c, Q, Kc, Vc, P, cap, nullptr, K, V, Y, n, hq, hkv, b, scale, ws,
                            ws_bytes);
}

int launch_prefix_paged_bf16(const Ctx& c, const void* Q, const void* Kpool, const void* Vpool,
                             const PagedCache& pg, const void* K, const void* V, void* Y, int n,
                             int hq, int hkv, int b, float scale, void* ws, size_t ws_bytes) {
  const int Pmax = pg.max_pages << pg.ps_log2;
  return launch_prefix_impl(c, Q, Kpool, Vpool, Pmax, Pmax, &pg, K, V, Y, n, hq, hkv, b, scale,
                            ws, ws_bytes);
}

}  // namespace bha
