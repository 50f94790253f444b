// bha_state_commit and bha_state_prefill, bf16 tensor-core path (d = 128).
//
// Both build the linear-attention prefix state of "Retrofitting Linear
// Attention into Diffusion Language Models" (worked example: S_1 =
// phi(K_1)^T V_1 and S_{1,2} = S_1 + phi(K_2)^T V_2, phi = ReLU):
//     S[r][c] (+)= sum_t relu(k_t[r]) v_t[c],   z[r] (+)= sum_t relu(k_t[r]).
// phi(K)^T V is an M=128 (feature r) x N=128 (value column c) contraction
// over tokens t, run on tcgen05 with both operands MN-major: the K and V
// tiles land by TMA exactly as they sit in memory ([t][128] rows, SW128),
// phi is applied in place, and the fp32 accumulator lives in TMEM.
//
// Commit: one CTA per (request, KV head): one MMA chain over the b block
// tokens gives phi(K)^T V in TMEM, which goes through a swizzled fp32 tile
// (thread = row r, conflict-free) to a TMA reduce-add into S (the add is
// done at L2, one 64-column half at a time): S never passes through the SM.
// The operands, S included, are prefetched into L2 before the kernel waits
// for the previous one.
//
// Prefill: one CTA per (unit, chunk of the prompt), a 3-stage TMA ring of
// 64-token K/V tiles (32 KB per stage) feeding the MMA warp; the chunk's
// partial state goes to the workspace (or straight to S when the prompt is
// one chunk) and a second kernel adds the chunks in a fixed order.
//
// Feature maps (the method details' kernel-function approximation): elu + 1
// is applied in place like ReLU (packed bf16 arithmetic, elu1_bf16x2).  The
// projected map phi(k) = ReLU(k W_g) takes one more MMA per K tile, the
// transposed projection (K W_g)^T = W_g^T K^T (M = 128 features, N =
// tokens, K = 128 inputs; A = W_g MN-major as it sits in memory, B = the K
// tile K-major), into spare TMEM columns; one thread per feature applies the
// ReLU, sums z, and writes phi(K)^T over the consumed K tile as a K-major
// operand for phi(K)^T V.
#include <cuda.h>
#include <cuda_runtime.h>

#include "bha_internal.h"
#include "bha_ptx.cuh"

namespace bha {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr uint32_t kSBytes = kD * kD * 4;   // 64 KB fp32 state tile
constexpr uint32_t kCtrlBytes = 128;

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

// Adds the TMEM accumulator (128 lanes x 128 fp32 columns) into / writes it
// over the swizzled fp32 state tile at `tile` (4 SW128 boxes of 128 rows x
// 32 columns).  Warp w handles rows 32*(w%4).., columns 64*(w/4)..
__device__ __forceinline__ void accum_to_tile(uint32_t tmem, uint32_t tile, int warp, int lane,
                                              bool add) {
  const int r = (warp & 3) * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
#pragma unroll 1
  for (int bx = 2 * (warp >> 2); bx < 2 * (warp >> 2) + 2; ++bx) {
    float acc[32];
    tmem_ld32_sync(tmem + lane_base + bx * 32, acc);
    const uint32_t row = tile + bx * 16384 + r * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t addr = row + ((j ^ (r & 7)) << 4);
      float4 v = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
      if (add) {
        const float4 s = ld_shared_f4(addr);
        v.x += s.x;
        v.y += s.y;
        v.z += s.z;
        v.w += s.w;
      }
      st_shared_f4(addr, v);
    }
  }
}

// Zeros in place of the accumulator (a chunk with no tokens): same tile
// addressing as accum_to_tile.
__device__ __forceinline__ void zero_tile(uint32_t tile, int warp, int lane) {
  const int r = (warp & 3) * 32 + lane;
#pragma unroll 1
  for (int bx = 2 * (warp >> 2); bx < 2 * (warp >> 2) + 2; ++bx) {
    const uint32_t row = tile + bx * 16384 + r * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) st_shared_f4(row + (j << 4), make_float4(0.f, 0.f, 0.f, 0.f));
  }
}

// ------------------------------------------------------------------ commit

struct CommitArgs {
  float* z;   // [units][128] or null
  int* err;
  int b;
  int hkv;    // unit u uses W[u % hkv] (projected map)
};

template <int BPAD>
struct CommitLayout {
  static constexpr uint32_t kKV = BPAD * 256;
  static constexpr uint32_t kOffS = 0;
  static constexpr uint32_t kOffK = kSBytes;
  static constexpr uint32_t kOffV = kOffK + kKV;
  static constexpr uint32_t kTiles = kOffV + kKV;
  static constexpr uint32_t kSmem = kTiles + 1024;
};

template <int BPAD, int FMAP>
__global__ void __launch_bounds__(kThreads, 2)
    k_commit_bf16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmS, const CommitArgs a) {
  using Lay = CommitLayout<BPAD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t ctrl = (base - raw >= kCtrlBytes) ? raw : base + Lay::kTiles;
  uint8_t* ctrl_ptr = smem_raw + (ctrl - raw);
  const uint32_t bar_kv = ctrl, bar_done = ctrl + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl_ptr + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl_ptr + 36);

  if (warp == 0) {
    if (lane == 0) {
      mbar_init(bar_kv, 1);
      mbar_init(bar_done, 1);
      *abort_flag = 0;
      fence_mbar_init();
      // warm L2 with this unit's operands while the previous kernel finishes
      tma_prefetch_l2_3d(&tmK, 0, 0, u);
      tma_prefetch_l2_3d(&tmK, 64, 0, u);
      tma_prefetch_l2_3d(&tmV, 0, 0, u);
      tma_prefetch_l2_3d(&tmV, 64, 0, u);
#pragma unroll
      for (int bx = 0; bx < 4; ++bx) tma_prefetch_l2_3d(&tmS, 32 * bx, 0, u);
    }
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  if (tid == 0) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_kv, 2 * Lay::kKV);
    tma_load_3d(base + Lay::kOffK, &tmK, bar_kv, 0, 0, u);
    tma_load_3d(base + Lay::kOffK + BPAD * 128, &tmK, bar_kv, 64, 0, u);
    tma_load_3d(base + Lay::kOffV, &tmV, bar_kv, 0, 0, u);
    tma_load_3d(base + Lay::kOffV + BPAD * 128, &tmV, bar_kv, 64, 0, u);
  }

  // phi(K) in place
  bool ok = warp_all(mbar_wait(bar_kv, 0, a.err, abort_flag));
  if (ok) {
    for (uint32_t v = tid; v < Lay::kKV / 16; v += kThreads) {
      const uint32_t addr = base + Lay::kOffK + v * 16;
      uint4 x = ld_shared_v4(addr);
      st_shared_v4(addr, phi_bf16x2<FMAP>(x.x), phi_bf16x2<FMAP>(x.y), phi_bf16x2<FMAP>(x.z),
                   phi_bf16x2<FMAP>(x.w));
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  if (tid == 32 && !*abort_flag) {
    // D[r][c] = sum_t phi(K)[t][r] V[t][c]: both operands MN-major SW128
    tc_fence_after();
    constexpr uint32_t idesc = make_idesc_bf16(128, 128, 1, 1);
#pragma unroll
    for (int ks = 0; ks < BPAD / 16; ++ks) {
      const uint64_t da = make_sdesc(base + Lay::kOffK + ks * 2048, BPAD * 128, 1024, kLayoutSW128);
      const uint64_t db = make_sdesc(base + Lay::kOffV + ks * 2048, BPAD * 128, 1024, kLayoutSW128);
      mma_bf16_ss(tmem, da, db, idesc, ks > 0 ? 1u : 0u);
    }
    mma_commit(bar_done);
  }

  // z += column sums of phi(K) (threads 0..127, one feature each)
  if (a.z != nullptr && tid < kD && !*abort_flag) {
    const int rr = tid;
    const uint32_t col = base + Lay::kOffK + (rr >> 6) * (BPAD * 128) + (rr & 7) * 2;
    float s = 0.f;
    for (int t = 0; t < a.b; ++t) {
      unsigned short hv;
      const uint32_t addr = col + t * 128 + (((((rr & 63) >> 3) ^ (t & 7))) << 4);
      asm volatile("ld.shared.u16 %0, [%1];" : "=h"(hv) : "r"(addr));
      s += __uint_as_float(static_cast<uint32_t>(hv) << 16);
    }
    a.z[static_cast<size_t>(u) * kD + rr] += s;
  }

  ok = warp_all(mbar_wait(bar_done, 0, a.err, abort_flag));
  tc_fence_after();
  if (ok) accum_to_tile(tmem, base + Lay::kOffS, warp, lane, false);
  fence_proxy_async_smem();
  tc_fence_before();
  // each 64-column half is added into S as soon as its four warps are done
  const int hb = warp >> 2;
  named_barrier_sync(1 + hb, 128);
  if ((tid & 127) == 0 && ok && !*abort_flag) {
    tma_reduce_add_3d(&tmS, base + Lay::kOffS + (2 * hb) * 16384, 64 * hb, 0, u);
    tma_reduce_add_3d(&tmS, base + Lay::kOffS + (2 * hb + 1) * 16384, 64 * hb + 32, 0, u);
    bulk_commit_group();
    bulk_wait_group_read0();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Commit under the projected map.  TMEM: phi(K)^T V at [0, 128), the
// projection (K W_g)^T at [128, 128 + BPAD).  Warps 0-3 (thread = feature r
// = TMEM lane) turn row r of the projection into row r of phi(K)^T.
template <int BPAD>
struct CommitProjLayout {
  static constexpr uint32_t kKV = BPAD * 256;
  static constexpr uint32_t kOffS = 0;
  static constexpr uint32_t kOffK = kSBytes;           // K, then phi(K)^T over it
  static constexpr uint32_t kOffV = kOffK + kKV;
  static constexpr uint32_t kOffW = kOffV + kKV;
  static constexpr uint32_t kTiles = kOffW + 32768;
  static constexpr uint32_t kSmem = kTiles + 1024;
  static constexpr uint32_t kRowB = 2 * BPAD;          // one phi(K)^T row: BPAD tokens
};

template <int BPAD>
__global__ void __launch_bounds__(kThreads, BPAD <= 32 ? 2 : 1)
    k_commit_proj_bf16(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmS,
                       const __grid_constant__ CUtensorMap tmW, const CommitArgs a) {
  using Lay = CommitProjLayout<BPAD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x, g = u % a.hkv;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t ctrl = (base - raw >= kCtrlBytes) ? raw : base + Lay::kTiles;
  uint8_t* ctrl_ptr = smem_raw + (ctrl - raw);
  const uint32_t bar_kv = ctrl, bar_done = ctrl + 16, bar_w = ctrl + 24,
                 bar_kw = ctrl + 40, bar_phik = ctrl + 48;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl_ptr + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl_ptr + 36);

  if (warp == 0) {
    if (lane == 0) {
      mbar_init(bar_kv, 1);
      mbar_init(bar_done, 1);
      mbar_init(bar_w, 1);
      mbar_init(bar_kw, 1);
      mbar_init(bar_phik, 128);
      *abort_flag = 0;
      fence_mbar_init();
      tma_prefetch_l2_3d(&tmK, 0, 0, u);
      tma_prefetch_l2_3d(&tmK, 64, 0, u);
      tma_prefetch_l2_3d(&tmV, 0, 0, u);
      tma_prefetch_l2_3d(&tmV, 64, 0, u);
#pragma unroll
      for (int bx = 0; bx < 4; ++bx) tma_prefetch_l2_3d(&tmS, 32 * bx, 0, u);
      tma_prefetch_l2_3d(&tmW, 0, 0, g);
      tma_prefetch_l2_3d(&tmW, 64, 0, g);
    }
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  if (tid == 0) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_kw = tmem + 128;
  pdl_wait();

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_kv, 2 * Lay::kKV);
    tma_load_3d(base + Lay::kOffK, &tmK, bar_kv, 0, 0, u);
    tma_load_3d(base + Lay::kOffK + BPAD * 128, &tmK, bar_kv, 64, 0, u);
    tma_load_3d(base + Lay::kOffV, &tmV, bar_kv, 0, 0, u);
    tma_load_3d(base + Lay::kOffV + BPAD * 128, &tmV, bar_kv, 64, 0, u);
    mbar_arrive_expect_tx(bar_w, 32768);
    tma_load_3d(base + Lay::kOffW, &tmW, bar_w, 0, 0, g);
    tma_load_3d(base + Lay::kOffW + 16384, &tmW, bar_w, 64, 0, g);
  }
  if (tid == 128) {
    // (K W_g)^T[r][t] = sum_i W_g[i][r] K[t][i]: A = W_g MN-major, B = K K-major
    if (mbar_wait(bar_kv, 0, a.err, abort_flag) && mbar_wait(bar_w, 0, a.err, abort_flag)) {
      tc_fence_after();
      constexpr uint32_t idesc = make_idesc_bf16(128, BPAD, 1, 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t da = make_sdesc(base + Lay::kOffW + ks * 2048, 16384, 1024, kLayoutSW128);
        const uint64_t db = make_sdesc(base + Lay::kOffK + (ks >> 2) * (BPAD * 128) + (ks & 3) * 32,
                                       16, 1024, kLayoutSW128);
        mma_bf16_ss(t_kw, da, db, idesc, ks > 0 ? 1u : 0u);
      }
      mma_commit(bar_kw);
    }
  }
  if (warp < 4) {
    // thread = feature r: ReLU, bf16, z, row r of phi(K)^T over the consumed K
    const int r = tid;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const bool okk = warp_all(mbar_wait(bar_kw, 0, a.err, abort_flag));
    tc_fence_after();
    if (okk) {
      float zs = 0.f;
#pragma unroll
      for (int j0 = 0; j0 < BPAD; j0 += 16) {
        float f[16];
        tmem_ld16_sync(t_kw + lane_base + j0, f);
        uint32_t w[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          w[q] = pack_bf16x2(fmaxf(f[2 * q], 0.f), fmaxf(f[2 * q + 1], 0.f));
          // padded tokens are zero rows of K, so their features are 0
          zs += __uint_as_float(w[q] << 16) + __uint_as_float(w[q] & 0xFFFF0000u);
        }
        st_shared_v4(kmajor_chunk<Lay::kRowB>(base + Lay::kOffK, r, j0 / 8), w[0], w[1], w[2], w[3]);
        st_shared_v4(kmajor_chunk<Lay::kRowB>(base + Lay::kOffK, r, j0 / 8 + 1), w[4], w[5], w[6],
                     w[7]);
      }
      if (a.z != nullptr) a.z[static_cast<size_t>(u) * kD + r] += zs;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(bar_phik);
  }
  if (tid == 128 && !*abort_flag) {
    // D[r][c] = sum_t phi(K)^T[r][t] V[t][c]: A K-major, B = V MN-major
    if (mbar_wait(bar_phik, 0, a.err, abort_flag)) {
      tc_fence_after();
      constexpr uint32_t idesc = make_idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int ks = 0; ks < BPAD / 16; ++ks) {
        const uint64_t da = make_sdesc(base + Lay::kOffK + ks * 32, 16, 8 * Lay::kRowB,
                                       kmajor_layout<Lay::kRowB>());
        const uint64_t db = make_sdesc(base + Lay::kOffV + ks * 2048, BPAD * 128, 1024, kLayoutSW128);
        mma_bf16_ss(tmem, da, db, idesc, ks > 0 ? 1u : 0u);
      }
      mma_commit(bar_done);
    }
  }

  const bool ok = warp_all(mbar_wait(bar_done, 0, a.err, abort_flag));
  tc_fence_after();
  if (ok) accum_to_tile(tmem, base + Lay::kOffS, warp, lane, false);
  fence_proxy_async_smem();
  tc_fence_before();
  const int hb = warp >> 2;
  named_barrier_sync(1 + hb, 128);
  if ((tid & 127) == 0 && ok && !*abort_flag) {
    tma_reduce_add_3d(&tmS, base + Lay::kOffS + (2 * hb) * 16384, 64 * hb, 0, u);
    tma_reduce_add_3d(&tmS, base + Lay::kOffS + (2 * hb + 1) * 16384, 64 * hb + 32, 0, u);
    bulk_commit_group();
    bulk_wait_group_read0();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------ prefill

constexpr int kTok = 64;                  // tokens per pipeline stage
constexpr int kStages = 3;
constexpr uint32_t kStageBytes = 2 * kTok * kD * 2;   // K + V tile: 32 KB
constexpr uint32_t kPrefTiles = kStages * kStageBytes; // 96 KB (>= 64 KB epilogue tile)
constexpr uint32_t kPrefSmem = kPrefTiles + 1024;
constexpr int kMaxTilesPerChunk = 64;     // 4096 tokens
constexpr int kMinTilesPerChunk = 16;     // 1024 tokens
constexpr int kTargetCtas = 296;          // two CTAs on each of 148 SMs

struct PrefillArgs {
  float* zdst;       // [items][128] or null (partial or final z)
  int* err;
  int T;             // prompt tokens (the longest, for ragged prompts)
  int splits;        // chunks per unit
  int tiles_per;     // 64-token tiles per chunk
  int hkv;           // unit u uses W[u % hkv] (projected map)
  const int* T_lens; // ragged prompts: [n] tokens per request (device), else null
};

// Prompt length of unit u's request: T, or its own length (clamped to
// [0, T]) for ragged prompts, whose rows past it are padding.  Reads device
// memory: call after pdl_wait.
__device__ __forceinline__ int unit_tokens(const PrefillArgs& a, int u) {
  return a.T_lens ? min(max(__ldg(a.T_lens + u / a.hkv), 0), a.T) : a.T;
}

template <int FMAP>
__global__ void __launch_bounds__(kThreads, 2)
    k_prefill_bf16(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmOut, const PrefillArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x;                // = u * splits + s
  const int u = item / a.splits, sp = item % a.splits;
  const int tile0 = sp * a.tiles_per;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t ctrl = (base - raw >= kCtrlBytes) ? raw : base + kPrefTiles;
  uint8_t* ctrl_ptr = smem_raw + (ctrl - raw);
  const uint32_t bar_full = ctrl, bar_relu = ctrl + 24, bar_empty = ctrl + 48,
                 bar_done = ctrl + 72;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl_ptr + 80);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl_ptr + 84);

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(bar_full + 8 * s, 1);
        mbar_init(bar_relu + 8 * s, 128);
        mbar_init(bar_empty + 8 * s, 1);
      }
      mbar_init(bar_done, 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  if (tid == 0) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  const int Tu = unit_tokens(a, u);
  const int ntile = max(0, min(a.tiles_per, (Tu + kTok - 1) / kTok - tile0));

  float zacc[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) zacc[q] = 0.f;

  if (tid == 0) {
    // producer
    for (int i = 0; i < ntile; ++i) {
      const int st = i % kStages;
      if (i >= kStages &&
          !mbar_wait(bar_empty + 8 * st, ((i / kStages) - 1) & 1, a.err, abort_flag))
        break;
      const uint32_t sbase = base + st * kStageBytes;
      const uint32_t bf = bar_full + 8 * st;
      const int t0 = (tile0 + i) * kTok;
      mbar_arrive_expect_tx(bf, kStageBytes);
      tma_load_3d(sbase, &tmK, bf, 0, t0, u);
      tma_load_3d(sbase + 8192, &tmK, bf, 64, t0, u);
      tma_load_3d(sbase + 16384, &tmV, bf, 0, t0, u);
      tma_load_3d(sbase + 24576, &tmV, bf, 64, t0, u);
    }
  } else if (tid == 32) {
    // MMA issuer: D[r][c] += sum_t phi(K)[t][r] V[t][c], both MN-major SW128
    constexpr uint32_t idesc = make_idesc_bf16(128, 128, 1, 1);
    bool ok = true;
    for (int i = 0; i < ntile && ok; ++i) {
      const int st = i % kStages;
      ok = mbar_wait(bar_relu + 8 * st, (i / kStages) & 1, a.err, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sbase = base + st * kStageBytes;
#pragma unroll
      for (int ks = 0; ks < kTok / 16; ++ks) {
        const uint64_t da = make_sdesc(sbase + ks * 2048, 8192, 1024, kLayoutSW128);
        const uint64_t db = make_sdesc(sbase + 16384 + ks * 2048, 8192, 1024, kLayoutSW128);
        mma_bf16_ss(tmem, da, db, idesc, (i | ks) ? 1u : 0u);
      }
      mma_commit(bar_empty + 8 * st);
    }
    if (ok) mma_commit(bar_done);
  } else if (warp >= 4) {
    // phi(K) in place; thread owns logical 16-byte column chunk (box, j) of
    // rows t_sub + 8k, so it can also accumulate z for those 8 features.
    const int w = tid - 128;
    const int box = w >> 6, j = (w >> 3) & 7, tsub = w & 7;
    for (int i = 0; i < ntile; ++i) {
      const int st = i % kStages;
      if (!mbar_wait(bar_full + 8 * st, (i / kStages) & 1, a.err, abort_flag)) break;
      const uint32_t kt = base + st * kStageBytes + box * 8192;
      // rows past the prompt: zero-filled past the buffer (ReLU keeps them
      // zero, elu + 1 would make them 1), padding of a ragged prompt inside
      // it (K and V cleared, so that 0 times V stays finite)
      const int tvalid = Tu - (tile0 + i) * kTok;
      const bool clear = FMAP != kFmapRelu || a.T_lens != nullptr;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int t = tsub + 8 * k;
        const uint32_t addr = kt + t * 128 + ((j ^ (t & 7)) << 4);
        uint4 x = ld_shared_v4(addr);
        x.x = phi_bf16x2<FMAP>(x.x);
        x.y = phi_bf16x2<FMAP>(x.y);
        x.z = phi_bf16x2<FMAP>(x.z);
        x.w = phi_bf16x2<FMAP>(x.w);
        if (clear && t >= tvalid) {
          x = make_uint4(0u, 0u, 0u, 0u);
          if (a.T_lens != nullptr) st_shared_v4(addr + 16384, 0u, 0u, 0u, 0u);   // V row
        }
        st_shared_v4(addr, x.x, x.y, x.z, x.w);
        const uint32_t wv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          zacc[2 * q] += __uint_as_float(wv[q] << 16);
          zacc[2 * q + 1] += __uint_as_float(wv[q] & 0xFFFF0000u);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_relu + 8 * st);
    }
  }

  // ---- epilogue: accumulator -> fp32 tile -> TMA store (partial or final).
  // A chunk past a ragged prompt's end stores nothing (the reduce reads only
  // the chunks its request has), or zeros when it is the unit's only chunk.
  __syncwarp();
  const bool store = ntile > 0 || a.splits == 1;
  const bool ok = warp_all(mbar_wait(bar_done, 0, a.err, abort_flag)) && store;
  tc_fence_after();
  if (ok) {
    if (ntile > 0)
      accum_to_tile(tmem, base, warp, lane, false);
    else
      zero_tile(base, warp, lane);
  }
  fence_proxy_async_smem();
  if (warp >= 4 && a.zdst != nullptr) {
    // reduce the 8 row-phases that share (box, j)
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      float v = zacc[q];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      zacc[q] = v;
    }
    const int w = tid - 128;
    const int box = w >> 6, j = (w >> 3) & 7, tsub = w & 7;
    if (tsub == 0 && ok) {
      float* zd = a.zdst + static_cast<size_t>(item) * kD + box * 64 + j * 8;
      reinterpret_cast<float4*>(zd)[0] = make_float4(zacc[0], zacc[1], zacc[2], zacc[3]);
      reinterpret_cast<float4*>(zd)[1] = make_float4(zacc[4], zacc[5], zacc[6], zacc[7]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && ok && !*abort_flag) {
#pragma unroll
    for (int bx = 0; bx < 4; ++bx) tma_store_3d(&tmOut, base + bx * 16384, 32 * bx, 0, item);
    bulk_commit_group();
    bulk_wait_group_read0();
  }
  __syncwarp();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Prefill under the projected map: the ReLU kernel's 3-stage ring and two
// CTAs per SM, with W_g^T, the A operand of the projection, held in TMEM
// (64 columns: lane = feature j, two bf16 inputs per column) so that shared
// memory holds only the K / V tiles.  TMEM: phi(K)^T V at [0, 128), W_g^T at
// [128, 192), one tile's projection (K W_g)^T at [192, 256).  The MMA thread
// issues tile i's projection once the feature writers have read tile
// i - 1's out of TMEM, and phi(K)^T V of tile i once its features are
// written; warps 4-7 (thread = feature r) read the projection, release it,
// apply the ReLU, add to z and write row r of phi(K)^T over the consumed K
// tile (K-major SW128, 64 tokens = 128 B).
struct PrefillProjArgs {
  PrefillArgs p;
  const uint16_t* W;   // [hkv][128][128] bf16 bits
};

__global__ void __launch_bounds__(kThreads, 2)
    k_prefill_proj_bf16(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmOut, const PrefillProjArgs pa) {
  const PrefillArgs& a = pa.p;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x;                // = u * splits + s
  const int u = item / a.splits, sp = item % a.splits;
  const int g = u % a.hkv;
  const int tile0 = sp * a.tiles_per;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t ctrl = (base - raw >= kCtrlBytes) ? raw : base + kPrefTiles;
  uint8_t* ctrl_ptr = smem_raw + (ctrl - raw);
  const uint32_t bar_full = ctrl, bar_relu = ctrl + 24, bar_empty = ctrl + 48,
                 bar_done = ctrl + 72, bar_kw = ctrl + 88, bar_kwfree = ctrl + 96,
                 bar_wt = ctrl + 104;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl_ptr + 80);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl_ptr + 84);

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(bar_full + 8 * s, 1);
        mbar_init(bar_relu + 8 * s, 128);
        mbar_init(bar_empty + 8 * s, 1);
      }
      mbar_init(bar_done, 1);
      mbar_init(bar_kw, 1);
      mbar_init(bar_kwfree, 128);
      mbar_init(bar_wt, 128);
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  if (tid == 0) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_w = tmem + 128, t_kw = tmem + 192;
  pdl_wait();
  const int Tu = unit_tokens(a, u);
  const int ntile = max(0, min(a.tiles_per, (Tu + kTok - 1) / kTok - tile0));

  float zacc = 0.f;
  if (tid == 0) {
    // producer
    for (int i = 0; i < ntile; ++i) {
      const int st = i % kStages;
      if (i >= kStages &&
          !mbar_wait(bar_empty + 8 * st, ((i / kStages) - 1) & 1, a.err, abort_flag))
        break;
      const uint32_t sbase = base + st * kStageBytes;
      const uint32_t bf = bar_full + 8 * st;
      const int t0 = (tile0 + i) * kTok;
      mbar_arrive_expect_tx(bf, kStageBytes);
      tma_load_3d(sbase, &tmK, bf, 0, t0, u);
      tma_load_3d(sbase + 8192, &tmK, bf, 64, t0, u);
      tma_load_3d(sbase + 16384, &tmV, bf, 0, t0, u);
      tma_load_3d(sbase + 24576, &tmV, bf, 64, t0, u);
    }
  } else if (tid == 32) {
    // (K W_g)^T of tile i: A = W_g^T from TMEM, B = the K tile (K-major)
    constexpr uint32_t id_kw = make_idesc_bf16(128, kTok, 0, 0);
    constexpr uint32_t id_sv = make_idesc_bf16(128, 128, 0, 1);
    auto issue_kw = [&](int i) -> bool {
      const int st = i % kStages;
      if (!mbar_wait(bar_full + 8 * st, (i / kStages) & 1, a.err, abort_flag)) return false;
      tc_fence_after();
      const uint32_t sbase = base + st * kStageBytes;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t db =
            make_sdesc(sbase + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kLayoutSW128);
        mma_bf16_ts(t_kw, t_w + 8 * ks, db, id_kw, ks > 0 ? 1u : 0u);
      }
      mma_commit(bar_kw);
      return true;
    };
    // phi(K)^T V of tile j into the accumulator: A K-major, B = V MN-major
    auto issue_sv = [&](int j) -> bool {
      const int sj = j % kStages;
      if (!mbar_wait(bar_relu + 8 * sj, (j / kStages) & 1, a.err, abort_flag)) return false;
      tc_fence_after();
      const uint32_t sb = base + sj * kStageBytes;
#pragma unroll
      for (int ks = 0; ks < kTok / 16; ++ks) {
        const uint64_t da = make_sdesc(sb + ks * 32, 16, 1024, kLayoutSW128);
        const uint64_t db = make_sdesc(sb + 16384 + ks * 2048, 8192, 1024, kLayoutSW128);
        mma_bf16_ss(tmem, da, db, id_sv, (j | ks) ? 1u : 0u);
      }
      mma_commit(bar_empty + 8 * sj);
      return true;
    };
    bool ok = mbar_wait(bar_wt, 0, a.err, abort_flag) && (ntile < 1 || issue_kw(0));
    for (int j = 0; j < ntile && ok; ++j) {
      if (j + 1 < ntile) {
        // the projection buffer is free once tile j's was read out of it
        ok = mbar_wait(bar_kwfree, j & 1, a.err, abort_flag) && issue_kw(j + 1);
        if (!ok) break;
      }
      ok = issue_sv(j);
    }
    if (ok) mma_commit(bar_done);
  } else if (warp >= 4) {
    const int r = tid - 128;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    {
      // W_g^T into TMEM: column c of lane r holds inputs 2c (low) and 2c + 1
      const uint16_t* Wg = pa.W + static_cast<size_t>(g) * kD * kD + r;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float f[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int i0 = 2 * (32 * h + c);
          const uint32_t lo = __ldg(Wg + i0 * kD), hi = __ldg(Wg + (i0 + 1) * kD);
          f[c] = __uint_as_float(lo | (hi << 16));
        }
        tmem_st32(t_w + lane_base + 32 * h, f);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_wt);
    }
    for (int i = 0; i < ntile; ++i) {
      const int st = i % kStages;
      if (!warp_all(mbar_wait(bar_kw, i & 1, a.err, abort_flag))) break;
      tc_fence_after();
      float f[64];
      tmem_ld32_sync(t_kw + lane_base, *reinterpret_cast<float(*)[32]>(f));
      tmem_ld32_sync(t_kw + lane_base + 32, *reinterpret_cast<float(*)[32]>(f + 32));
      tc_fence_before();
      mbar_arrive(bar_kwfree);
      const uint32_t kt = base + st * kStageBytes;   // phi(K)^T over the consumed K tile
      // tokens past the prompt: zero rows of K past the buffer (features 0);
      // padding of a ragged prompt inside it: features and V rows cleared
      const int tvalid = a.T_lens != nullptr ? Tu - (tile0 + i) * kTok : kTok;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = 8 * c + 2 * q;
          w[q] = pack_bf16x2(t < tvalid ? fmaxf(f[t], 0.f) : 0.f,
                             t + 1 < tvalid ? fmaxf(f[t + 1], 0.f) : 0.f);
          zacc += __uint_as_float(w[q] << 16) + __uint_as_float(w[q] & 0xFFFF0000u);
        }
        st_shared_v4(kmajor_chunk<128>(kt, r, c), w[0], w[1], w[2], w[3]);
      }
      for (int idx = r; idx < (kTok - max(tvalid, 0)) * 16; idx += 128) {
        const int row = tvalid + (idx >> 4), ch = idx & 15;
        st_shared_v4(kt + 16384 + (ch >> 3) * 8192 + row * 128 + (ch & 7) * 16, 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      mbar_arrive(bar_relu + 8 * st);
    }
  }

  // ---- epilogue: accumulator -> fp32 tile -> TMA store (partial or final);
  // nothing for a chunk past a ragged prompt's end unless it is the only one
  __syncwarp();
  const bool store = ntile > 0 || a.splits == 1;
  const bool ok = warp_all(mbar_wait(bar_done, 0, a.err, abort_flag)) && store;
  tc_fence_after();
  if (ok) {
    if (ntile > 0)
      accum_to_tile(tmem, base, warp, lane, false);
    else
      zero_tile(base, warp, lane);
  }
  fence_proxy_async_smem();
  if (warp >= 4 && a.zdst != nullptr && ok)
    a.zdst[static_cast<size_t>(item) * kD + (tid - 128)] = zacc;
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && ok && !*abort_flag) {
#pragma unroll
    for (int bx = 0; bx < 4; ++bx) tma_store_3d(&tmOut, base + bx * 16384, 32 * bx, 0, item);
    bulk_commit_group();
    bulk_wait_group_read0();
  }
  __syncwarp();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// S[u] = sum over chunks s (in order) of ws_S[u][s];  same for z.  Ragged
// prompts: only the chunks the request's prompt reaches (none: S = z = 0).
struct ReduceArgs {
  int splits;
  const int* T_lens;   // ragged: [n] prompt tokens, else null
  int hkv, T, tiles_per;
};

__global__ void __launch_bounds__(256) k_prefill_reduce(const float4* __restrict__ wsS,
                                                        const float4* __restrict__ wsZ,
                                                        float4* __restrict__ S,
                                                        float4* __restrict__ z,
                                                        const ReduceArgs ra) {
  pdl_launch_dependents();
  pdl_wait();
  const int u = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;    // float4 index within a unit
  constexpr int kS4 = kD * kD / 4, kZ4 = kD / 4;
  const int splits = ra.splits;
  int nvalid = splits;
  if (ra.T_lens != nullptr) {
    const int Tu = min(max(__ldg(ra.T_lens + u / ra.hkv), 0), ra.T);
    nvalid = min(splits, ((Tu + kTok - 1) / kTok + ra.tiles_per - 1) / ra.tiles_per);
  }
  if (e < kS4) {
    const float4* p = wsS + static_cast<size_t>(u) * splits * kS4 + e;
    float4 acc = nvalid > 0 ? p[0] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 1; s < nvalid; ++s) {
      const float4 v = p[static_cast<size_t>(s) * kS4];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    S[static_cast<size_t>(u) * kS4 + e] = acc;
  }
  if (z != nullptr && e < kZ4) {
    const float4* p = wsZ + static_cast<size_t>(u) * splits * kZ4 + e;
    float4 acc = nvalid > 0 ? p[0] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 1; s < nvalid; ++s) {
      const float4 v = p[static_cast<size_t>(s) * kZ4];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    z[static_cast<size_t>(u) * kZ4 + e] = acc;
  }
}

// Chunking of a T-token prompt: chunks of at most 64 tiles (4096 tokens),
// split further (down to 16 tiles) while there are fewer than two CTAs per
// SM of a 148-SM part.  Depends only on (units, T), so the workspace query
// and the launch always agree.
void prefill_plan(int units, int T, int* splits, int* tiles_per) {
  const int tiles = (T + kTok - 1) / kTok;
  int s = (tiles + kMaxTilesPerChunk - 1) / kMaxTilesPerChunk;
  if (units * s < kTargetCtas) {
    const int want = (kTargetCtas + units - 1) / units;
    const int cap = (tiles + kMinTilesPerChunk - 1) / kMinTilesPerChunk;
    const int more = want < cap ? want : cap;
    if (more > s) s = more;
  }
  if (s < 1) s = 1;
  const int tp = (tiles + s - 1) / s;
  *splits = (tiles + tp - 1) / tp;   // no empty chunk
  *tiles_per = tp;
}

bool state_tmap(CUtensorMap* m, const float* S, uint64_t items) {
  const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)kD, items};
  const uint64_t strides[2] = {kD * 4ull, (uint64_t)kD * kD * 4ull};
  const uint32_t box[3] = {32, 128, 1};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, S, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

bool tokens_tmap(CUtensorMap* m, const void* X, int T, int units, uint32_t box_rows) {
  const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)T, (uint64_t)units};
  const uint64_t strides[2] = {kD * 2ull, (uint64_t)T * kD * 2ull};
  const uint32_t box[3] = {64, box_rows, 1};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, X, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

bool weights_tmap(CUtensorMap* m, const void* W, int hkv) {
  const uint64_t dims[3] = {(uint64_t)kD, (uint64_t)kD, (uint64_t)hkv};
  const uint64_t strides[2] = {kD * 2ull, (uint64_t)kD * kD * 2ull};
  const uint32_t box[3] = {64, (uint32_t)kD, 1};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, W, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int BPAD, int FMAP>
int launch_commit_cfg(const Ctx& c, const CUtensorMap& tk, const CUtensorMap& tv,
                      const CUtensorMap& ts, const CUtensorMap& tw, const CommitArgs& a,
                      int units) {
  if constexpr (FMAP == kFmapReluProj) {
    using Lay = CommitProjLayout<BPAD>;
    auto kern = k_commit_proj_bf16<BPAD>;
    static Prepared prepared;
    if (!prepare_kernel(c, kern, (int)Lay::kSmem, prepared)) return -5;
    return launch_pdl(kern, units, kThreads, Lay::kSmem, c.stream, tk, tv, ts, tw, a);
  } else {
    using Lay = CommitLayout<BPAD>;
    auto kern = k_commit_bf16<BPAD, FMAP>;
    static Prepared prepared;
    if (!prepare_kernel(c, kern, (int)Lay::kSmem, prepared)) return -5;
    return launch_pdl(kern, units, kThreads, Lay::kSmem, c.stream, tk, tv, ts, a);
  }
}

template <int BPAD>
int launch_commit_bpad(const Ctx& c, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& ts, const CUtensorMap& tw, const CommitArgs& a,
                       int units, int fmap) {
  switch (fmap) {
    case kFmapRelu: return launch_commit_cfg<BPAD, kFmapRelu>(c, tk, tv, ts, tw, a, units);
    case kFmapElu1: return launch_commit_cfg<BPAD, kFmapElu1>(c, tk, tv, ts, tw, a, units);
    default: return launch_commit_cfg<BPAD, kFmapReluProj>(c, tk, tv, ts, tw, a, units);
  }
}

}  // namespace

int launch_commit_bf16(const Ctx& c, const void* K, const void* V, int units, int b, float* S,
                       float* z, int fmap, const void* W, int hkv) {
  const int bpad = b <= 16 ? 16 : (b <= 32 ? 32 : 64);
  CUtensorMap tk, tv, ts, tw;
  if (!tokens_tmap(&tk, K, b, units, bpad) || !tokens_tmap(&tv, V, b, units, bpad) ||
      !state_tmap(&ts, S, units))
    return -5;
  if (fmap == kFmapReluProj) {
    if (!weights_tmap(&tw, W, hkv)) return -5;
  } else {
    tw = tk;
  }
  CommitArgs a{z, c.dev_err, b, hkv};
  switch (bpad) {
    case 16: return launch_commit_bpad<16>(c, tk, tv, ts, tw, a, units, fmap);
    case 32: return launch_commit_bpad<32>(c, tk, tv, ts, tw, a, units, fmap);
    default: return launch_commit_bpad<64>(c, tk, tv, ts, tw, a, units, fmap);
  }
}

size_t prefill_bf16_workspace(int units, int T) {
  if (T <= 0 || units <= 0) return 0;
  int splits, tp;
  prefill_plan(units, T, &splits, &tp);
  if (splits <= 1) return 0;
  return static_cast<size_t>(units) * splits * (kD * kD + kD) * sizeof(float);
}

int launch_prefill_bf16(const Ctx& c, const void* K, const void* V, int units, int T, float* S,
                        float* z, void* ws, size_t ws_bytes, int fmap, const void* W, int hkv,
                        const int* T_lens) {
  if (T == 0) {
    if (cudaMemsetAsync(S, 0, static_cast<size_t>(units) * kD * kD * 4, c.stream) != cudaSuccess)
      return -5;
    if (z && cudaMemsetAsync(z, 0, static_cast<size_t>(units) * kD * 4, c.stream) != cudaSuccess)
      return -5;
    return 0;
  }
  int splits, tp;
  prefill_plan(units, T, &splits, &tp);
  const size_t need = prefill_bf16_workspace(units, T);
  if (need > ws_bytes) return -4;
  float* outS = S;
  float* outZ = z;
  if (splits > 1) {
    outS = static_cast<float*>(ws);
    outZ = z ? outS + static_cast<size_t>(units) * splits * kD * kD : nullptr;
  }
  CUtensorMap tk, tv, to;
  if (!tokens_tmap(&tk, K, T, units, kTok) || !tokens_tmap(&tv, V, T, units, kTok) ||
      !state_tmap(&to, outS, static_cast<uint64_t>(units) * splits))
    return -5;
  PrefillArgs a{outZ, c.dev_err, T, splits, tp, hkv, T_lens};
  int rc;
  if (fmap == kFmapReluProj) {
    static Prepared prepared_p;
    if (!prepare_kernel(c, k_prefill_proj_bf16, (int)kPrefSmem, prepared_p)) return -5;
    const PrefillProjArgs pa{a, static_cast<const uint16_t*>(W)};
    rc = launch_pdl(k_prefill_proj_bf16, units * splits, kThreads, kPrefSmem, c.stream, tk, tv,
                    to, pa);
  } else if (fmap == kFmapElu1) {
    static Prepared prepared_e;
    if (!prepare_kernel(c, k_prefill_bf16<kFmapElu1>, (int)kPrefSmem, prepared_e)) return -5;
    rc = launch_pdl(k_prefill_bf16<kFmapElu1>, units * splits, kThreads, kPrefSmem, c.stream, tk,
                    tv, to, a);
  } else {
    static Prepared prepared_r;
    if (!prepare_kernel(c, k_prefill_bf16<kFmapRelu>, (int)kPrefSmem, prepared_r)) return -5;
    rc = launch_pdl(k_prefill_bf16<kFmapRelu>, units * splits, kThreads, kPrefSmem, c.stream, tk,
                    tv, to, a);
  }
  if (rc) return -5;
  if (splits > 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((kD * kD / 4 + 255) / 256, units);
    cfg.blockDim = dim3(256);
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const ReduceArgs ra{splits, T_lens, hkv, T, tp};
    if (cudaLaunchKernelEx(&cfg, k_prefill_reduce, reinterpret_cast<const float4*>(outS),
                           reinterpret_cast<const float4*>(outZ), reinterpret_cast<float4*>(S),
                           reinterpret_cast<float4*>(z), ra) != cudaSuccess)
      return -5;
    if (cudaGetLastError() != cudaSuccess) return -5;
  }
  return 0;
}

}  // namespace bha
