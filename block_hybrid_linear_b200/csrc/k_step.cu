// bha_hybrid_step, bf16 tensor-core path for sm_100a (d = 128).
//
// One denoising step of block-hybrid attention ("Retrofitting Linear
// Attention into Diffusion Language Models", core formula; worked example,
// blocks 2 and 3):
//     y_i = sum_j softmax_j(scale q_i . k_j) v_j + phi(q_i) S,   phi = ReLU.
//
// One CTA per (request n, KV head g, 128-row tile of the G*b query rows that
// share g).  All operands of the unit are fetched by TMA at once:
//   Q   128 x 128 bf16  (2 SW128 boxes, K-major)       32 KB
//   S   128 x 128 fp32  (8 boxes of 32 x 64)           64 KB
//   K,V BPAD x 128 bf16 (2 SW128 boxes each)           2 x 8 KB at BPAD=32
// and the three contractions run on the 5th-generation tensor cores with
// fp32 accumulators in tensor memory (TMEM):
//   scores = Q K^T              M=128 N=BPAD K=128   -> TMEM cols [128,128+BPAD)
//   lin    = phi(Q) S_hi + phi(Q) S_lo   M=128 N=128 K=128 -> TMEM cols [0,128)
//   soft   = P V                M=128 N=128 K=BPAD   -> TMEM cols [128,256)
// S is fp32 in memory; each warp splits its 8 x 64 block in place into a bf16
// high part and a bf16 residual (S = S_hi + S_lo to ~2^-17 relative), so the
// state keeps ~16 mantissa bits on the bf16 tensor path.  phi(Q) is applied
// in place on the Q tile after the score MMA has read it; P (unnormalised
// softmax weights, <= 1) overwrites the K tile after the score MMA.  Each
// row-owner thread (warps 4-7, one TMEM lane each) does the row softmax in
// registers and the epilogue y = alpha * lin + beta * soft, and the bf16
// tile goes back by TMA store.  Shared memory is 113 KB at BPAD = 32 so two
// CTAs fit on one SM: the grid's loads are all in flight from the start.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "bha_internal.h"
#include "bha_ptx.cuh"

namespace bha {
namespace {

constexpr int kD = 128;
constexpr int kMT = 128;         // query rows per CTA (UMMA M)
constexpr int kThreads = 256;
constexpr uint32_t kQBytes = kMT * kD * 2;   // 32 KB
constexpr uint32_t kSBytes = kD * kD * 4;    // 64 KB
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffS = kQBytes;
constexpr uint32_t kOffK = kQBytes + kSBytes;
constexpr uint32_t kCtrlBytes = 128;

struct StepArgs {
  const float* z;     // [units][128] (shared mode)
  int* err;           // device error word
  int rows;           // G * b query rows per unit
  int b;              // active block length
  int mtiles;         // ceil(rows / 128)
  float scale;        // softmax scale
  float scale_log2;   // scale * log2(e)
  int shared;         // BHA_FLAG_SHARED_DENOM
};

template <int BPAD>
struct StepLayout {
  static constexpr uint32_t kKV = BPAD * 256;           // one of K / V (2 boxes)
  static constexpr uint32_t kOffV = kOffK + kKV;
  static constexpr uint32_t kTiles = kOffV + kKV;
  static constexpr uint32_t kSmem = kTiles + 1024;      // + alignment slack / ctrl
  static constexpr uint32_t kRowB = 2 * BPAD;           // bytes of one P row
  static constexpr uint32_t kPLayout = BPAD == 16 ? kLayoutSW32 : BPAD == 32 ? kLayoutSW64
                                                                           : kLayoutSW128;
};

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

template <int BPAD>
__global__ void __launch_bounds__(kThreads, BPAD <= 32 ? 2 : 1)
    k_step_bf16(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                const __grid_constant__ CUtensorMap tmY, const StepArgs a) {
  using Lay = StepLayout<BPAD>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int u = blockIdx.x / a.mtiles, mt = blockIdx.x % a.mtiles;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t ctrl = (base - raw >= kCtrlBytes) ? raw : base + Lay::kTiles;
  uint8_t* ctrl_ptr = smem_raw + (ctrl - raw);
  const uint32_t bar_q = ctrl, bar_k = ctrl + 8, bar_s = ctrl + 16, bar_v = ctrl + 48,
                 bar_sc = ctrl + 56, bar_p = ctrl + 64, bar_done = ctrl + 72;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl_ptr + 80);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl_ptr + 84);

  if (warp == 0) {
    if (lane == 0) {
      mbar_init(bar_q, 1);
      mbar_init(bar_k, 1);
      for (int c = 0; c < 4; ++c) mbar_init(bar_s + 8 * c, 1);
      mbar_init(bar_v, 1);
      mbar_init(bar_sc, 1);
      mbar_init(bar_p, 128);
      mbar_init(bar_done, 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_lin = tmem, t_soft = tmem + 128;

  // ---- producer: every operand of the unit in flight at once
  if (tid == 0) {
    const int row0 = mt * kMT;
    mbar_arrive_expect_tx(bar_q, kQBytes);
    tma_load_3d(base + kOffQ, &tmQ, bar_q, 0, row0, u);
    tma_load_3d(base + kOffQ + 16384, &tmQ, bar_q, 64, row0, u);
    mbar_arrive_expect_tx(bar_k, Lay::kKV);
    tma_load_3d(base + kOffK, &tmK, bar_k, 0, 0, u);
    tma_load_3d(base + kOffK + BPAD * 128, &tmK, bar_k, 64, 0, u);
    for (int c = 0; c < 4; ++c) {
      mbar_arrive_expect_tx(bar_s + 8 * c, 16384);
      tma_load_3d(base + kOffS + c * 16384, &tmS, bar_s + 8 * c, 0, 32 * c, u);
      tma_load_3d(base + kOffS + c * 16384 + 8192, &tmS, bar_s + 8 * c, 64, 32 * c, u);
    }
    mbar_arrive_expect_tx(bar_v, Lay::kKV);
    tma_load_3d(base + Lay::kOffV, &tmV, bar_v, 0, 0, u);
    tma_load_3d(base + Lay::kOffV + BPAD * 128, &tmV, bar_v, 64, 0, u);
  }

  // ---- MMA 1: scores = Q K^T  (both K-major SW128)
  if (tid == 32) {
    bool ok = mbar_wait(bar_q, 0, a.err, abort_flag) && mbar_wait(bar_k, 0, a.err, abort_flag);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = make_idesc_bf16(128, BPAD, 0, 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t da =
            make_sdesc(base + kOffQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128);
        const uint64_t db = make_sdesc(base + kOffK + (ks >> 2) * (BPAD * 128) + (ks & 3) * 32,
                                       16, 1024, kLayoutSW128);
        mma_bf16_ss(t_soft, da, db, idesc, ks > 0 ? 1u : 0u);
      }
      mma_commit(bar_sc);
    }
  }

  // ---- S (fp32) -> S_hi / S_lo (bf16, MN-major SW128 atoms), in place.
  // Warp w owns, in chunk c (rows 32c..32c+31), the 8 x 64 block at column
  // atom w/4, row group w%4: 2 KB of fp32 become a 1 KB S_hi atom followed
  // by a 1 KB S_lo atom.  Reads finish (syncwarp) before any write.
  bool ok = true;
  {
    const uint32_t colatom = warp >> 2, grp = warp & 3;
    for (int c = 0; c < 4; ++c) {
      ok = warp_all(ok && mbar_wait(bar_s + 8 * c, 0, a.err, abort_flag));
      if (!ok) break;
      const uint32_t blk = base + kOffS + c * 16384 + colatom * 8192 + grp * 2048;
      float4 x[4];
#pragma unroll
      for (int s = 0; s < 4; ++s) x[s] = ld_shared_f4(blk + (lane + 32 * s) * 16);
      __syncwarp();
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int f = lane + 32 * s;
        const int kr = f >> 4, n0 = (f & 15) * 4;
        const int j = n0 >> 3, half = (n0 >> 2) & 1;
        const uint32_t off = kr * 128 + ((j ^ kr) << 4) + half * 8;
        const __nv_bfloat16 h0 = __float2bfloat16_rn(x[s].x), h1 = __float2bfloat16_rn(x[s].y);
        const __nv_bfloat16 h2 = __float2bfloat16_rn(x[s].z), h3 = __float2bfloat16_rn(x[s].w);
        const float l0 = x[s].x - __bfloat162float(h0), l1 = x[s].y - __bfloat162float(h1);
        const float l2 = x[s].z - __bfloat162float(h2), l3 = x[s].w - __bfloat162float(h3);
        const uint32_t hi01 = (uint32_t)__bfloat16_as_ushort(h0) |
                              ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        const uint32_t hi23 = (uint32_t)__bfloat16_as_ushort(h2) |
                              ((uint32_t)__bfloat16_as_ushort(h3) << 16);
        st_shared_v2(blk + off, hi01, hi23);
        st_shared_v2(blk + 1024 + off, pack_bf16x2(l0, l1), pack_bf16x2(l2, l3));
      }
    }
  }
  fence_proxy_async_smem();

  // ---- wait for the score MMA, then phi(Q) in place and scores to registers
  ok = warp_all(ok && mbar_wait(bar_sc, 0, a.err, abort_flag));
  tc_fence_after();
  float sc[BPAD];
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  if (warp >= 4 && ok) {
#pragma unroll
    for (int j = 0; j < BPAD; j += 16) {
      float t[16];
      tmem_ld16_sync(t_soft + lane_base + j, t);
#pragma unroll
      for (int q = 0; q < 16; ++q) sc[j + q] = t[q];
    }
  }
  if (ok) {
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint32_t addr = base + kOffQ + (tid + kThreads * s) * 16;
      uint4 v = ld_shared_v4(addr);
      v.x = relu_bf16x2(v.x);
      v.y = relu_bf16x2(v.y);
      v.z = relu_bf16x2(v.z);
      v.w = relu_bf16x2(v.w);
      st_shared_v4(addr, v.x, v.y, v.z, v.w);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---- MMA 2: lin = phi(Q) S_hi + phi(Q) S_lo  (B MN-major SW128)
  if (tid == 32 && !*abort_flag) {
    tc_fence_after();
    constexpr uint32_t idesc = make_idesc_bf16(128, 128, 0, 1);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint64_t da =
            make_sdesc(base + kOffQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, kLayoutSW128);
        const uint32_t sb = base + kOffS + (ks >> 1) * 16384 + (ks & 1) * 4096 + part * 1024;
        const uint64_t db = make_sdesc(sb, 8192, 2048, kLayoutSW128);
        mma_bf16_ss(t_lin, da, db, idesc, (part | ks) ? 1u : 0u);
      }
    }
  }

  // ---- row softmax (warps 4-7: thread = query row = TMEM lane)
  float alpha = 1.f, beta = 0.f;
  const int r = (warp & 3) * 32 + lane;
  if (warp >= 4) {
    if (!*abort_flag) {
      float m = -INFINITY;
#pragma unroll
      for (int j = 0; j < BPAD; ++j) {
        if (j >= a.b) sc[j] = -INFINITY;
        m = fmaxf(m, sc[j]);
      }
      float l = 0.f;
#pragma unroll
      for (int j = 0; j < BPAD; ++j) {
        sc[j] = exp2f((sc[j] - m) * a.scale_log2);
        l += sc[j];
      }
      // P row r -> K region (K-major, swizzle width = row bytes)
      const uint32_t prow = base + kOffK + (r >> 3) * (8 * Lay::kRowB) + (r & 7) * Lay::kRowB;
      const uint32_t swz = Lay::kRowB == 128 ? (r & 7) : Lay::kRowB == 64 ? ((r & 7) >> 1)
                                                                          : ((r & 7) >> 2);
#pragma unroll
      for (int jj = 0; jj < BPAD / 8; ++jj) {
        st_shared_v4(prow + ((jj ^ swz) << 4), pack_bf16x2(sc[8 * jj + 0], sc[8 * jj + 1]),
                     pack_bf16x2(sc[8 * jj + 2], sc[8 * jj + 3]),
                     pack_bf16x2(sc[8 * jj + 4], sc[8 * jj + 5]),
                     pack_bf16x2(sc[8 * jj + 6], sc[8 * jj + 7]));
      }
      if (!a.shared) {
        alpha = 1.f;
        beta = 1.f / l;
      } else {
        // phi(q) . z from the row's phi(Q) (already ReLU'd in place)
        const float* zu = a.z + static_cast<size_t>(u) * kD;
        float qz = 0.f;
#pragma unroll
        for (int box = 0; box < 2; ++box) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 v = ld_shared_v4(base + kOffQ + box * 16384 + r * 128 +
                                         ((j ^ (r & 7)) << 4));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float lo = __uint_as_float(w[q] << 16);
              const float hi = __uint_as_float(w[q] & 0xFFFF0000u);
              qz = fmaf(lo, __ldg(zu + box * 64 + j * 8 + 2 * q), qz);
              qz = fmaf(hi, __ldg(zu + box * 64 + j * 8 + 2 * q + 1), qz);
            }
          }
        }
        // y = (sum e v + e^{-m_s} lin) / (l + e^{-m_s} qz),  m_s = scale * m,
        // evaluated without overflow for either sign of m_s.
        if (m >= 0.f) {
          const float em = exp2f(-m * a.scale_log2);
          const float inv = 1.f / (l + em * qz);
          alpha = em * inv;
          beta = inv;
        } else {
          const float t = exp2f(m * a.scale_log2);
          const float inv = 1.f / (t * l + qz);
          alpha = inv;
          beta = t * inv;
        }
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(bar_p);
  }

  // ---- MMA 3: soft = P V  (A K-major swizzled by row width, B MN-major SW128)
  if (tid == 32) {
    const bool ok3 = mbar_wait(bar_p, 0, a.err, abort_flag) &&
                     mbar_wait(bar_v, 0, a.err, abort_flag);
    if (ok3) {
      tc_fence_after();
      constexpr uint32_t idesc = make_idesc_bf16(128, 128, 0, 1);
#pragma unroll
      for (int ks = 0; ks < BPAD / 16; ++ks) {
        const uint64_t da =
            make_sdesc(base + kOffK + ks * 32, 16, 8 * Lay::kRowB, Lay::kPLayout);
        const uint64_t db =
            make_sdesc(base + Lay::kOffV + ks * 2048, BPAD * 128, 1024, kLayoutSW128);
        mma_bf16_ss(t_soft, da, db, idesc, ks > 0 ? 1u : 0u);
      }
      mma_commit(bar_done);
    }
  }

  // ---- epilogue: y = alpha * lin + beta * soft -> bf16 tile (SW128) in Q's place
  if (warp >= 4) {
    const bool okd = warp_all(mbar_wait(bar_done, 0, a.err, abort_flag));
    tc_fence_after();
    if (okd) {
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float lin[32], soft[32];
        tmem_ld32_sync(t_lin + lane_base + cc * 32, lin);
        tmem_ld32_sync(t_soft + lane_base + cc * 32, soft);
        const uint32_t row = base + kOffQ + (cc >> 1) * 16384 + r * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int j = (cc & 1) * 4 + q;
          const int e = 8 * q;
          st_shared_v4(row + ((j ^ (r & 7)) << 4),
                       pack_bf16x2(fmaf(alpha, lin[e + 0], beta * soft[e + 0]),
                                   fmaf(alpha, lin[e + 1], beta * soft[e + 1])),
                       pack_bf16x2(fmaf(alpha, lin[e + 2], beta * soft[e + 2]),
                                   fmaf(alpha, lin[e + 3], beta * soft[e + 3])),
                       pack_bf16x2(fmaf(alpha, lin[e + 4], beta * soft[e + 4]),
                                   fmaf(alpha, lin[e + 5], beta * soft[e + 5])),
                       pack_bf16x2(fmaf(alpha, lin[e + 6], beta * soft[e + 6]),
                                   fmaf(alpha, lin[e + 7], beta * soft[e + 7])));
        }
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    if (!*abort_flag) {
      tma_store_3d(&tmY, base + kOffQ, 0, mt * kMT, u);
      tma_store_3d(&tmY, base + kOffQ + 16384, 64, mt * kMT, u);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }
  __syncwarp();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int BPAD>
int launch_bpad(const Ctx& c, const CUtensorMap& tq, const CUtensorMap& tk,
                const CUtensorMap& tv, const CUtensorMap& ts, const CUtensorMap& ty,
                const StepArgs& a, int grid) {
  using Lay = StepLayout<BPAD>;
  auto kern = k_step_bf16<BPAD>;
  static std::atomic<uint64_t> prepared{0};
  if (!prepare_kernel(kern, (int)Lay::kSmem, prepared)) return -5;
  kern<<<grid, kThreads, Lay::kSmem, c.stream>>>(tq, tk, tv, ts, ty, a);
  return cudaGetLastError() == cudaSuccess ? 0 : -5;
}

}  // namespace

int launch_step_bf16(const Ctx& c, const void* Q, const void* K, const void* V, const float* S,
                     const float* z, void* Y, int n, int hq, int hkv, int b, float scale,
                     int shared) {
  const int G = hq / hkv;
  const int rows = G * b;
  const int units = n * hkv;
  const int bpad = b <= 16 ? 16 : (b <= 32 ? 32 : 64);
  const int mtiles = (rows + kMT - 1) / kMT;

  CUtensorMap tq, tk, tv, ts, ty;
  const uint64_t dq[3] = {(uint64_t)kD, (uint64_t)rows, (uint64_t)units};
  const uint64_t sq[2] = {kD * 2ull, (uint64_t)rows * kD * 2ull};
  const uint32_t bq[3] = {64, kMT, 1};
  const uint64_t dk[3] = {(uint64_t)kD, (uint64_t)b, (uint64_t)units};
  const uint64_t sk[2] = {kD * 2ull, (uint64_t)b * kD * 2ull};
  const uint32_t bk[3] = {64, (uint32_t)bpad, 1};
  const uint64_t ds[3] = {(uint64_t)kD, (uint64_t)kD, (uint64_t)units};
  const uint64_t ss[2] = {kD * 4ull, (uint64_t)kD * kD * 4ull};
  const uint32_t bs[3] = {64, 32, 1};
  if (!encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Q, dq, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Y, dq, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, K, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, S, ds, ss, bs,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return -5;

  StepArgs a;
  a.z = z;
  a.err = c.dev_err;
  a.rows = rows;
  a.b = b;
  a.mtiles = mtiles;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.shared = shared;
  const int grid = units * mtiles;
  switch (bpad) {
    case 16: return launch_bpad<16>(c, tq, tk, tv, ts, ty, a, grid);
    case 32: return launch_bpad<32>(c, tq, tk, tv, ts, ty, a, grid);
    default: return launch_bpad<64>(c, tq, tk, tv, ts, ty, a, grid);
  }
}

}  // namespace bha
