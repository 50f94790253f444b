// bha_hybrid_step, bf16 tensor-core path for sm_100a (d = 128).
//
// One denoising step of block-hybrid attention ("Retrofitting Linear
// Attention into Diffusion Language Models", core formula; worked example,
// blocks 2 and 3):
//     y_i = sum_j softmax_j(scale q_i . k_j) v_j + phi(q_i) S,   phi = ReLU
// (the worked example's map), elu + 1, or ReLU after a per-KV-head d x d
// projection W_g (the method details' kernel-function approximation).
//
// One CTA per (request n, KV head g, 128-row tile of the G*b query rows that
// share g); on grids of at most one CTA per SM, two CTAs per tile, each
// computing half of the output columns (HALF, below).  TMA brings Q, K, V
// first; the fp32 state S (four 32-row chunks) is requested once this CTA's
// Q has landed, so that across the grid the softmax operands are not queued
// behind the state (measured: 2 % faster in the default mode, 4 % with the
// shared denominator); column halves outside the fused commit request it
// with Q (EARLY, below):
//   Q   128 x 128 bf16  (2 SW128 boxes, K-major)               32 KB
//   S   128 x 128 fp32  (16 boxes of 32 rows x 32 cols, 32B-atom swizzle)  64 KB
//   K,V BPAD x 128 bf16 (2 SW128 boxes each)                   2 x 8 KB at BPAD=32
// Work (TMEM columns: D = [0,128), the scores in its first BPAD columns until
// P V overwrites them; phi(Q) = [128,256)):
//   MMA (bf16)  scores = Q K^T                    M=128 N=BPAD K=128
//   warps 0-3 (thread = query row = TMEM lane): phi(q) as fp32 into TMEM
//   warps 4-7 (likewise): row softmax in registers, P -> smem over the
//        consumed K tile
//   MMA (bf16)  D  = P V                          M=128 N=128 K=BPAD
//   MMA (tf32)  D += phi(Q)[TMEM] S[smem]  per state chunk, as it lands
//   all 8 warps: D -> bf16 -> swizzled tile -> TMA store, per 64-column half
// The fp32 state is consumed by the tensor core as it lands: no conversion
// pass over it (tf32 keeps 10 of its 23 mantissa bits in the products; the
// accumulation is fp32).  In the default mode P is normalised before P V; with
// the shared denominator the row's e^{-m} goes into phi(q) or P (whichever
// keeps it <= 1) and the epilogue applies 1 / denominator.  Shared memory is
// 113 KB at BPAD = 32, so two CTAs share an SM and the grid's loads are all
// in flight from the start.  Launched with programmatic dependent launch: the
// prologue, including L2 prefetches of all operands, overlaps the previous
// kernel's tail.
//
// Projected map phi(q) = ReLU(q W_g): one more MMA (bf16) Q W_g -> TMEM,
// M=128 N=128 K=128, into the columns phi(Q) occupies, then the ReLU in
// TMEM.  W_g (32 KB, from L2: every unit of KV head g reads the
// same W_g) lands where state chunks 2-3 go; those two chunks are loaded
// once the Q W_g product has read it, so shared memory and the two CTAs per
// SM stay as they are.
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
constexpr uint32_t kOffW = kOffS + kSBytes / 2;   // projected map: over state chunks 2-3
constexpr uint32_t kCtrlBytes = 256;
// Shared denominator: largest log2 scale put into P instead of phi(q) (P <=
// 2^92, its row sum <= 64 * 2^92: far inside fp32 and bf16 range).
constexpr float kSharedShiftLog2 = 92.f;

struct StepArgs {
  const float* z;     // [units][128] (shared mode)
  const float* lpre;  // reuse: [units][rows] cached prefix log-normalisers (natural log)
  float* zc;          // [units][128] updated by the fused commit, or null
  int* err;           // device error word
  int hkv;            // KV heads (unit u uses W[u % hkv])
  int rows;           // G * b query rows per unit
  int b;              // active block length
  int mtiles;         // ceil(rows / 128)
  float scale;        // softmax scale
  float scale_log2;   // scale * log2(e)
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

// z[k] of the 128-vector spread over a warp (lane l holds z[4l .. 4l+3]);
// k is a compile-time index, every lane calls it.
__device__ __forceinline__ float z_at(float4 zl, int k) {
  const float c = (k & 3) == 0 ? zl.x : (k & 3) == 1 ? zl.y : (k & 3) == 2 ? zl.z : zl.w;
  return __shfl_sync(0xffffffffu, c, k >> 2);
}

// phi(q_r) as fp32 into TMEM (this thread's lane, columns [0, 128) from
// `tcol`), read from row r of the SW128 Q tile; one wait for all four
// 32-column stores.  Elementwise maps only (phi of a bf16 pair is a bf16
// pair; the tensor core reads the values as tf32).  QZ: also returns
// phi(q_r) . z (the shared denominator's term); lane l holds z[4l .. 4l+3].
template <int FMAP, bool QZ>
__device__ __forceinline__ float write_phiq(uint32_t qtile, int r, uint32_t tcol, float4 zl) {
  float qz[4] = {0.f, 0.f, 0.f, 0.f};   // four independent partial sums
#pragma unroll
  for (int cg = 0; cg < 4; ++cg) {
    float f[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = (cg & 1) * 4 + q;
      const uint4 v = ld_shared_v4(qtile + (cg >> 1) * 16384 + r * 128 + ((j ^ (r & 7)) << 4));
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t p2 = phi_bf16x2<FMAP>(w4[e]);
        f[8 * q + 2 * e] = __uint_as_float(p2 << 16);
        f[8 * q + 2 * e + 1] = __uint_as_float(p2 & 0xFFFF0000u);
      }
    }
    tmem_st32(tcol + cg * 32, f);
    if (QZ) {
#pragma unroll
      for (int e = 0; e < 32; ++e) qz[e & 3] = fmaf(f[e], z_at(zl, cg * 32 + e), qz[e & 3]);
    }
  }
  tmem_wait_st();
  return (qz[0] + qz[1]) + (qz[2] + qz[3]);
}

// phi(q_r) . z from phi(q_r) as written to TMEM (this thread's lane, 128
// columns from `tcol`): the same values and the same four partial sums, in
// the same order, as write_phiq<FMAP, true>, read back after phi(Q) has been
// handed to the tensor core so that the products need not wait for them.
__device__ __forceinline__ float qz_from_tmem(uint32_t tcol, float4 zl) {
  float qz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int cg = 0; cg < 4; ++cg) {
    float f[32];
    tmem_ld32_sync(tcol + cg * 32, f);
#pragma unroll
    for (int e = 0; e < 32; ++e) qz[e & 3] = fmaf(f[e], z_at(zl, cg * 32 + e), qz[e & 3]);
  }
  return (qz[0] + qz[1]) + (qz[2] + qz[3]);
}

// Projected map: the Q W_g product sits in TMEM (this thread's lane, 128
// columns from `tcol`); replace it by max(., 0).  QZ: also returns
// phi(q_r) . z (z spread over the lanes as for write_phiq).
template <bool QZ>
__device__ __forceinline__ float relu_tmem_phiq(uint32_t tcol, float4 zl) {
  // the same four partial sums, in the same order, as write_phiq
  float qz[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int cg = 0; cg < 4; ++cg) {
    float f[32];
    tmem_ld32_sync(tcol + cg * 32, f);
#pragma unroll
    for (int q = 0; q < 32; ++q) f[q] = fmaxf(f[q], 0.f);
    tmem_st32(tcol + cg * 32, f);
    if (QZ) {
#pragma unroll
      for (int q = 0; q < 32; ++q) qz[q & 3] = fmaf(f[q], z_at(zl, cg * 32 + q), qz[q & 3]);
    }
  }
  tmem_wait_st();
  return (qz[0] + qz[1]) + (qz[2] + qz[3]);
}

// Shared denominator: this thread's row of phi(Q) in TMEM times s.
__device__ __forceinline__ void scale_tmem_row(uint32_t tcol, float s) {
#pragma unroll
  for (int cg = 0; cg < 4; ++cg) {
    float f[32];
    tmem_ld32_sync(tcol + cg * 32, f);
#pragma unroll
    for (int q = 0; q < 32; ++q) f[q] *= s;
    tmem_st32(tcol + cg * 32, f);
  }
  tmem_wait_st();
}

// COMMIT with the projected map: the transposed projection (K W_g)^T =
// W_g^T K^T (A = W_g MN-major, B = K K-major, M = 128 features, N = BPAD
// tokens) is issued with Q W_g into the accumulator's columns [BPAD,
// 2 BPAD), which P V overwrites only after warps 0-3 (thread = feature)
// have read it; they write phi(K)^T as a K-major operand over the consumed
// K tile.
// COMMIT: also fold this step's block into the state after using it (the
// block's last denoising step): S += phi(K)^T V, z += sum_t phi(k_t); the
// state is read once (the tile the step used) and phi(K)^T V goes over that
// tile to a TMA reduce-add into S.  P then lives in the consumed Q tile so that K survives for the commit MMA,
// and phi(K)^T V accumulates in the TMEM columns phi(Q) used.  Default mode
// and a single 128-row tile per unit only.
// HALF (small grids): a pair of adjacent CTAs shares a unit, each computing
// 64 of the 128 output columns: it loads the whole Q and K (the pair's second
// reads hit L2) but only its half of V and of every state chunk, and runs
// P V and phi(Q) S at N = 64.  The scores and the softmax are computed by
// both.  This doubles the CTAs of a grid that would leave most SMs idle.
// With the fused commit each CTA adds its half of phi(K)^T V to S, and the
// first of the pair adds the block's sum of phi(k) to z.
// REUSE (the exact path with reuse for stable tokens, LoSA page, cache
// reuse and technical details): the "state" tile is this 128-row tile's
// cached prefix outputs O_pre (fp32, one row per query row, normalised) and
// no phi(Q) S product runs; the row owners also compute the block's
// log-normaliser and, with the row's cached prefix log-normaliser, the
// online-softmax weights a, b (a + b = 1), and the epilogue writes
// y = a (P V) + b O_pre.
template <int BPAD, bool SHARED, bool COMMIT, int FMAP, bool HALF, bool REUSE = false>
__global__ void __launch_bounds__(kThreads, BPAD <= 32 ? 2 : 1)
    k_step_bf16(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmW,
                const StepArgs a) {
  static_assert(!(SHARED && COMMIT), "the fused commit runs in the default mode only");
  static_assert(!(REUSE && (SHARED || COMMIT || FMAP != kFmapRelu)),
                "the reuse block pass has no state, commit or feature map");
  constexpr bool PROJ = FMAP == kFmapReluProj;
  static_assert(!(HALF && PROJ), "column halves: elementwise maps only");
  constexpr int kN = HALF ? 64 : 128;                   // output columns of this CTA
  // Column halves in the default mode (small grids, latency bound): the
  // state is requested with Q, the scores sit in the accumulator's unused
  // upper half, and tid 0 (once phi(Q) is in) issues the phi(Q) S products
  // as the state lands, then P V, while the row owners run the softmax.
  // With the shared denominator the products go first only when no row of
  // the tile moves e^{-m} into its phi(q) (the row owners say so on bar_m
  // once their row maxima are known); otherwise P V goes first and the
  // products follow the rows' rescaling, as in the whole-unit order.
  constexpr bool EARLY = HALF && !COMMIT && !REUSE;
  constexpr uint32_t kChunkS = HALF ? 8192 : 16384;     // bytes of one state chunk here
  using Lay = StepLayout<BPAD>;
  // P (the softmax weights, bf16, K-major) goes over the consumed K tile, or
  // over the consumed Q tile when K is still needed by the commit
  constexpr uint32_t kOffP = COMMIT ? kOffQ : kOffK;
  extern __shared__ __align__(1024) uint8_t smem_raw[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = HALF ? static_cast<int>(blockIdx.x & 1u) : 0;   // column half
  const int item = HALF ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int u = item / a.mtiles, mt = item % a.mtiles;
  const int g = u % a.hkv;
  // first row of this tile in the state-shaped operand: the d x d state, or
  // (reuse) this tile's rows of the cached prefix outputs
  const int srow0 = REUSE ? mt * kMT : 0;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t ctrl = (base - raw >= kCtrlBytes) ? raw : base + Lay::kTiles;
  uint8_t* ctrl_ptr = smem_raw + (ctrl - raw);
  const uint32_t bar_q = ctrl, bar_k = ctrl + 8, bar_v = ctrl + 16, bar_s = ctrl + 24,
                 bar_sc = ctrl + 56, bar_p = ctrl + 64, bar_a = ctrl + 72, bar_done = ctrl + 80,
                 bar_phik = ctrl + 96, bar_ds = ctrl + 104, bar_w = ctrl + 112,
                 bar_qw = ctrl + 120, bar_kwr = ctrl + 128, bar_a2 = ctrl + 136,
                 bar_qz = ctrl + 144, bar_m = ctrl + 160;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctrl_ptr + 88);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctrl_ptr + 92);
  // shared denominator: set by a row owner whose row scales its phi(q) (row
  // max past the shift bound), before it arrives on bar_p
  volatile int* rescale_flag = reinterpret_cast<volatile int*>(ctrl_ptr + 152);

  if (warp == 0) {
    if (lane == 0) {
      mbar_init(bar_q, 1);
      mbar_init(bar_k, 1);
      mbar_init(bar_v, 1);
      for (int c = 0; c < 4; ++c) mbar_init(bar_s + 8 * c, 1);
      mbar_init(bar_sc, 1);
      mbar_init(bar_p, 128);
      mbar_init(bar_a, 128);
      if (SHARED) {
        mbar_init(bar_a2, 128);
        mbar_init(bar_qz, 128);
        if (EARLY) mbar_init(bar_m, 128);
        *rescale_flag = 0;
      }
      mbar_init(bar_done, 1);
      if (COMMIT) {
        mbar_init(bar_phik, 128);
        mbar_init(bar_ds, 1);
      }
      if (PROJ) {
        mbar_init(bar_w, 1);
        mbar_init(bar_qw, 1);
        if (COMMIT) mbar_init(bar_kwr, 128);
      }
      *abort_flag = 0;
      fence_mbar_init();
      tma_prefetch_desc(&tmY);
      // Warm L2 with every operand of the unit while the previous kernel of
      // the stream finishes (the loads proper wait for it, see pdl_wait).
      const int row0 = mt * kMT;
      tma_prefetch_l2_3d(&tmQ, 0, row0, u);
      tma_prefetch_l2_3d(&tmQ, 64, row0, u);
      tma_prefetch_l2_3d(&tmK, 0, 0, u);
      tma_prefetch_l2_3d(&tmK, 64, 0, u);
      for (int vb = 0; vb < 2; ++vb)
        if (!HALF || vb == half) tma_prefetch_l2_3d(&tmV, 64 * vb, 0, u);
      for (int c = 0; c < 4; ++c)
        for (int nb = 0; nb < 4; ++nb)
          if (!HALF || (nb >> 1) == half) tma_prefetch_l2_3d(&tmS, 32 * nb, srow0 + 32 * c, u);
      if (PROJ) {
        tma_prefetch_l2_3d(&tmW, 0, 0, g);
        tma_prefetch_l2_3d(&tmW, 64, 0, g);
      }
      if (SHARED)
        for (int l = 0; l < 4; ++l) prefetch_l2(a.z + static_cast<size_t>(u) * kD + 32 * l);
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
  const uint32_t t_d = tmem;           // [0, 128): the output accumulator
  const uint32_t t_a = tmem + 128;     // [128, 256): phi(Q) as tf32 (the MMA's A)
  // Scores sit in the accumulator's first columns (P V overwrites them once
  // read), so phi(Q) is built in parallel.  With the shared denominator,
  // warps 0-3 hand each row's phi(q) . z to the row owners through that
  // row's own bytes of the consumed Q tile (row r of Q is read by thread r
  // alone, and by the MMAs that bar_sc / bar_qw complete).
  const uint32_t t_sc = EARLY ? t_d + 64 : t_d;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  pdl_wait();   // inputs may come from the previous kernel of the stream

  // chunk c = state rows 32c..32c+31; box (c, nb) = its columns 32nb..32nb+31
  // (HALF: only the half's two boxes of every chunk, packed)
  auto load_state_chunks = [&](int c0, int c1) {
    for (int c = c0; c < c1; ++c) {
      mbar_arrive_expect_tx(bar_s + 8 * c, kChunkS);
#pragma unroll
      for (int nn = 0; nn < kN / 32; ++nn) {
        const int nb = HALF ? 2 * half + nn : nn;
        tma_load_3d(base + kOffS + c * kChunkS + nn * 4096, &tmS, bar_s + 8 * c, 32 * nb,
                    srow0 + 32 * c, u);
      }
    }
  };

  // ---- producer: Q, K, V first (the softmax half); the state chunks are
  // requested once this CTA's Q has landed (below), so that across the grid
  // the softmax operands are not queued behind the state
  if (tid == 0) {
    const int row0 = mt * kMT;
    mbar_arrive_expect_tx(bar_q, kQBytes);
    tma_load_3d(base + kOffQ, &tmQ, bar_q, 0, row0, u);
    tma_load_3d(base + kOffQ + 16384, &tmQ, bar_q, 64, row0, u);
    mbar_arrive_expect_tx(bar_k, Lay::kKV);
    tma_load_3d(base + kOffK, &tmK, bar_k, 0, 0, u);
    tma_load_3d(base + kOffK + BPAD * 128, &tmK, bar_k, 64, 0, u);
    if (HALF) {
      mbar_arrive_expect_tx(bar_v, Lay::kKV / 2);
      tma_load_3d(base + Lay::kOffV, &tmV, bar_v, 64 * half, 0, u);
    } else {
      mbar_arrive_expect_tx(bar_v, Lay::kKV);
      tma_load_3d(base + Lay::kOffV, &tmV, bar_v, 0, 0, u);
      tma_load_3d(base + Lay::kOffV + BPAD * 128, &tmV, bar_v, 64, 0, u);
    }
    if (PROJ) {
      mbar_arrive_expect_tx(bar_w, 2 * 16384);
      tma_load_3d(base + kOffW, &tmW, bar_w, 0, 0, g);
      tma_load_3d(base + kOffW + 16384, &tmW, bar_w, 64, 0, g);
    }
    // the projected map's state chunks 0-1 (2-3 follow over W_g)
    if (PROJ) load_state_chunks(0, 2);
    if (EARLY) load_state_chunks(0, 4);
  }

  float beta = 1.f;   // per-row output scale (shared denominator only)
  // reuse: the row's weights of P V and of its cached prefix output
  float ralpha = 1.f, rbeta = 0.f;
  if (REUSE && warp < 4) {
    // only the cached prefix rows to request, once Q has landed
    const bool okq = warp_all(mbar_wait(bar_q, 0, a.err, abort_flag));
    if (okq && lane == 0) load_state_chunks(warp, warp + 1);
  } else if (warp < 4) {
    // phi(q) for row r = 32 w + lane into TMEM as soon as Q has landed, in
    // parallel with the score MMA and the softmax (and phi(q) . z)
    // z (shared denominator), four values a lane, requested before Q lands
    float4 zl = make_float4(0.f, 0.f, 0.f, 0.f);
    if (SHARED) zl = __ldg(reinterpret_cast<const float4*>(a.z + static_cast<size_t>(u) * kD) + lane);
    float qz = 0.f;
    bool okf;
    if (PROJ) {
      okf = warp_all(mbar_wait(bar_qw, 0, a.err, abort_flag));
      tc_fence_after();
      if (okf && tid == 0) load_state_chunks(2, 4);
      if (okf) qz = relu_tmem_phiq<SHARED>(t_a + lane_base, zl);
    } else {
      okf = warp_all(mbar_wait(bar_q, 0, a.err, abort_flag));
      // state chunk w from warp w: the issue cost is spread over the warps
      // that build phi(Q), which the phi(Q) S products wait for
      if (!EARLY && okf && lane == 0) load_state_chunks(warp, warp + 1);
      // shared denominator: phi(q) . z along the way with column halves
      // (their products wait for it, see issue_early), read back from TMEM
      // once phi(Q) is handed over otherwise (the products need not wait)
      if (okf) qz = write_phiq<FMAP, SHARED && HALF>(base + kOffQ, warp * 32 + lane, t_a + lane_base, zl);
    }
    tc_fence_before();
    mbar_arrive(bar_a);   // phi(Q) is in TMEM
    if (SHARED && !HALF && !PROJ && okf) qz = qz_from_tmem(t_a + lane_base, zl);
    auto issue_early = [&]() {
      // the four state chunks' products as they land (the state was
      // requested with Q, so it usually lands before P is ready), then P V:
      // a fixed order, so that the result does not depend on timing
      bool ok3 = mbar_wait(bar_a, 0, a.err, abort_flag);
      bool late = false;   // shared denominator: some row rescales its phi(q)
      if (SHARED && ok3) {
        ok3 = mbar_wait(bar_m, 0, a.err, abort_flag);
        late = ok3 && *rescale_flag != 0;
      }
      auto products = [&](bool acc) {
        for (int c = 0; c < 4 && ok3; ++c) {
          ok3 = mbar_wait(bar_s + 8 * c, 0, a.err, abort_flag);
          if (!ok3) break;
          tc_fence_after();
          constexpr uint32_t idesc = make_idesc_tf32(128, kN, 0, 1);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t db = make_sdesc(base + kOffS + c * kChunkS + kk * 1024, 4096, 512,
                                           kLayoutSW128_32B);
            mma_tf32_ts(t_d, t_a + 32 * c + 8 * kk, db, idesc, (acc || c || kk) ? 1u : 0u);
          }
        }
      };
      auto pv = [&](bool acc) {
        ok3 = ok3 && mbar_wait(bar_p, 0, a.err, abort_flag) && mbar_wait(bar_v, 0, a.err, abort_flag);
        if (!ok3) return;
        tc_fence_after();
        constexpr uint32_t idesc = make_idesc_bf16(128, kN, 0, 1);
#pragma unroll
        for (int ks = 0; ks < BPAD / 16; ++ks) {
          const uint64_t da = make_sdesc(base + kOffP + ks * 32, 16, 8 * Lay::kRowB, Lay::kPLayout);
          const uint64_t db =
              make_sdesc(base + Lay::kOffV + ks * 2048, BPAD * 128, 1024, kLayoutSW128);
          mma_bf16_ss(t_d, da, db, idesc, (acc || ks) ? 1u : 0u);
        }
      };
      if (!late) {
        products(false);
        pv(true);
      } else {
        // the rescaled phi(q) rows are in TMEM once bar_a2 completes
        pv(false);
        ok3 = ok3 && mbar_wait(bar_a2, 0, a.err, abort_flag);
        products(true);
      }
      if (ok3) mma_commit(bar_done);
    };
    if (EARLY && !SHARED && tid == 0) issue_early();
    if (SHARED) {
      // phi(q) . z to the row owners, over row tid of the Q tile once the
      // score MMA (or, projected, Q W_g) has read it
      if (okf && (PROJ || warp_all(mbar_wait(bar_sc, 0, a.err, abort_flag))))
        st_shared_f32(base + kOffQ + tid * 128, qz);
      mbar_arrive(bar_qz);
      if (EARLY && tid == 0) issue_early();
    }
    if (COMMIT && PROJ) {
      // thread = feature r: row r of (K W_g)^T (landed with Q W_g) out of
      // TMEM, which P V may then overwrite; ReLU, bf16, z, and row r of
      // phi(K)^T over the consumed K tile
      constexpr uint32_t kRowB = 2 * BPAD;
      const int rr = tid;
      uint32_t wv[BPAD / 2];
      float zs = 0.f;
#pragma unroll
      for (int j0 = 0; j0 < BPAD; j0 += 16) {
        float f[16];
        tmem_ld16_sync(t_d + BPAD + lane_base + j0, f);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          // padded tokens are zero rows of K, so their features are 0
          wv[j0 / 2 + q] = pack_bf16x2(fmaxf(f[2 * q], 0.f), fmaxf(f[2 * q + 1], 0.f));
          zs += __uint_as_float(wv[j0 / 2 + q] << 16) +
                __uint_as_float(wv[j0 / 2 + q] & 0xFFFF0000u);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_kwr);
#pragma unroll
      for (int jj = 0; jj < BPAD / 8; ++jj)
        st_shared_v4(kmajor_chunk<kRowB>(base + kOffK, rr, jj), wv[4 * jj], wv[4 * jj + 1],
                     wv[4 * jj + 2], wv[4 * jj + 3]);
      fence_proxy_async_smem();
      mbar_arrive(bar_phik);
      if (a.zc != nullptr) a.zc[static_cast<size_t>(u) * kD + rr] += zs;
    } else if (COMMIT) {
      // phi(K) in place once the score MMA has read K, and this block's
      // column sums of phi(K) for z (thread = feature r)
      const bool okk = warp_all(mbar_wait(bar_sc, 0, a.err, abort_flag));
      if (okk) {
        for (uint32_t v = tid; v < Lay::kKV / 16; v += 128) {
          const uint32_t addr = base + kOffK + v * 16;
          const uint4 x = ld_shared_v4(addr);
          st_shared_v4(addr, phi_bf16x2<FMAP>(x.x), phi_bf16x2<FMAP>(x.y),
                       phi_bf16x2<FMAP>(x.z), phi_bf16x2<FMAP>(x.w));
        }
      }
      fence_proxy_async_smem();
      named_barrier_sync(4, 128);   // the whole phi(K) tile is written
      mbar_arrive(bar_phik);
      if (okk && a.zc != nullptr && half == 0) {
        const int rr = tid;
        const uint32_t col = base + kOffK + (rr >> 6) * (BPAD * 128) + (rr & 7) * 2;
        float zs = 0.f;
        for (int t = 0; t < a.b; ++t) {
          unsigned short hv;
          const uint32_t addr = col + t * 128 + ((((rr & 63) >> 3) ^ (t & 7)) << 4);
          asm volatile("ld.shared.u16 %0, [%1];" : "=h"(hv) : "r"(addr));
          zs += __uint_as_float(static_cast<uint32_t>(hv) << 16);
        }
        a.zc[static_cast<size_t>(u) * kD + rr] += zs;
      }
    }
  }
  if (warp >= 4) {
    // ---- row owners: thread = query row r of the tile = TMEM lane r
    const int r = (warp - 4) * 32 + lane;
    // reuse: the row's cached prefix log-normaliser (rows past the unit's:
    // none), read before the scores land
    float lp2 = -INFINITY;
    if (REUSE && mt * kMT + r < a.rows)
      lp2 = __ldg(a.lpre + static_cast<size_t>(u) * a.rows + mt * kMT + r) * 1.4426950408889634f;
    if (tid == 128) {
      if (mbar_wait(bar_q, 0, a.err, abort_flag) && mbar_wait(bar_k, 0, a.err, abort_flag)) {
        tc_fence_after();
        constexpr uint32_t idesc = make_idesc_bf16(128, BPAD, 0, 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t da = make_sdesc(base + kOffQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16,
                                         1024, kLayoutSW128);
          const uint64_t db = make_sdesc(base + kOffK + (ks >> 2) * (BPAD * 128) + (ks & 3) * 32,
                                         16, 1024, kLayoutSW128);
          mma_bf16_ss(t_sc, da, db, idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar_sc);
        if (PROJ && mbar_wait(bar_w, 0, a.err, abort_flag)) {
          // Q W_g: A = Q (K-major), B = W_g [input i][feature j] (MN-major)
          tc_fence_after();
          constexpr uint32_t idw = make_idesc_bf16(128, 128, 0, 1);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t da = make_sdesc(base + kOffQ + (ks >> 2) * 16384 + (ks & 3) * 32, 16,
                                           1024, kLayoutSW128);
            const uint64_t db = make_sdesc(base + kOffW + ks * 2048, 16384, 1024, kLayoutSW128);
            mma_bf16_ss(t_a, da, db, idw, ks > 0 ? 1u : 0u);
          }
          if (COMMIT) {
            // (K W_g)^T: A = W_g MN-major, B = K K-major
            constexpr uint32_t idk = make_idesc_bf16(128, BPAD, 1, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint64_t da = make_sdesc(base + kOffW + ks * 2048, 16384, 1024, kLayoutSW128);
              const uint64_t db = make_sdesc(
                  base + kOffK + (ks >> 2) * (BPAD * 128) + (ks & 3) * 32, 16, 1024, kLayoutSW128);
              mma_bf16_ss(t_d + BPAD, da, db, idk, ks > 0 ? 1u : 0u);
            }
          }
          mma_commit(bar_qw);
        }
      }
    }
    const bool ok = warp_all(mbar_wait(bar_sc, 0, a.err, abort_flag));
    tc_fence_after();
    float ascale = 1.f;
    // shared denominator: the row max in log2 units, the row sum, P's factor
    float m2 = 0.f, lsum = 1.f, pscale = 1.f;
    if (ok) {
      float sc[BPAD];
#pragma unroll
      for (int j = 0; j < BPAD; j += 16) {
        float t[16];
        tmem_ld16_sync(t_sc + lane_base + j, t);
#pragma unroll
        for (int q = 0; q < 16; ++q) sc[j + q] = t[q];
      }
      // keys past the block (padding of the MMA's N)
      if (a.b < BPAD) {
#pragma unroll
        for (int j = 0; j < BPAD; ++j)
          if (j >= a.b) sc[j] = -INFINITY;
      }
      float m4[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
      for (int j = 4; j < BPAD; j += 4) {
#pragma unroll
        for (int q = 0; q < 4; ++q) m4[q] = fmaxf(m4[q], sc[j + q]);
      }
      const float m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      // e_j = 2^{s_j scale log2 e - m scale log2 e}, on the packed fp32 pipe
      const float2 sl = make_float2(a.scale_log2, a.scale_log2);
      const float2 nb = make_float2(-m * a.scale_log2, -m * a.scale_log2);
      float2 l4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
#pragma unroll
      for (int j = 0; j < BPAD; j += 2) {
        float2 x = fma2(make_float2(sc[j], sc[j + 1]), sl, nb);
        x.x = ex2_sfu(x.x);
        x.y = ex2_sfu(x.y);
        sc[j] = x.x;
        sc[j + 1] = x.y;
        l4[(j >> 1) & 3] = add2(l4[(j >> 1) & 3], x);
      }
      const float2 l2 = add2(add2(l4[0], l4[1]), add2(l4[2], l4[3]));
      const float l = l2.x + l2.y;
      if (SHARED) {
        // y = (sum_j e^{s_j - c} v_j + e^{-c} phi(q) S) / (sum_j e^{s_j - c} +
        // e^{-c} phi(q).z) for any c; e_j = e^{s_j - m_s} above, m_s = scale * m.
        // c = 0 (P = e_j e^{m_s}, phi(q) as it is) while 2^kSharedShiftLog2
        // bounds P; past that c = m_s and e^{-m_s} goes into phi(q) in TMEM
        // below.  P depends on the scores alone, so P V never waits for
        // phi(Q); only the output's 1 / denominator needs phi(q) . z.
        m2 = m * a.scale_log2;
        pscale = m2 > kSharedShiftLog2 ? 1.f : exp2f(m2);
        lsum = l;
        if (m2 > kSharedShiftLog2) *rescale_flag = 1;   // before this row's bar_p arrive
        if (EARLY) mbar_arrive(bar_m);
      } else {
        pscale = 1.f / l;   // default: P is normalised, the terms add as they are
      }
      if (REUSE) {
        // online-softmax merge of the block part (log2-normaliser lb2) with
        // the cached prefix part (lp2): y = wb/(wp+wb) o_b + wp/(wp+wb) o_p
        const float lb2 = m * a.scale_log2 + __log2f(l);
        const float M2 = fmaxf(lp2, lb2);
        const float wp = exp2f(lp2 - M2), wb = exp2f(lb2 - M2);
        const float inv = 1.f / (wp + wb);
        ralpha = wb * inv;
        rbeta = wp * inv;
      }
      // P row r (K-major, swizzle width = row bytes); over the Q tile only
      // once phi(Q) has been read out of it
      if (COMMIT) mbar_wait(bar_a, 0, a.err, abort_flag);
      const uint32_t prow = base + kOffP + (r >> 3) * (8 * Lay::kRowB) + (r & 7) * Lay::kRowB;
      const uint32_t swz = Lay::kRowB == 128 ? (r & 7) : Lay::kRowB == 64 ? ((r & 7) >> 1)
                                                                          : ((r & 7) >> 2);
      const float2 ps = make_float2(pscale, pscale);
#pragma unroll
      for (int jj = 0; jj < BPAD / 8; ++jj) {
        const float* e = sc + 8 * jj;
        const float2 p0 = mul2(make_float2(e[0], e[1]), ps), p1 = mul2(make_float2(e[2], e[3]), ps),
                     p2 = mul2(make_float2(e[4], e[5]), ps), p3 = mul2(make_float2(e[6], e[7]), ps);
        st_shared_v4(prow + ((jj ^ swz) << 4), pack_bf16x2(p0.x, p0.y), pack_bf16x2(p1.x, p1.y),
                     pack_bf16x2(p2.x, p2.y), pack_bf16x2(p3.x, p3.y));
      }
    }
    if (SHARED && EARLY && !ok) mbar_arrive(bar_m);
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(bar_p);

    // MMA issuer (a row owner too): P V as soon as P and V are in, before
    // its own row's shared-denominator work below
    bool ok2 = true;
    if (!EARLY && tid == 128) {
      ok2 = mbar_wait(bar_p, 0, a.err, abort_flag) && mbar_wait(bar_v, 0, a.err, abort_flag) &&
            (!(COMMIT && PROJ) || mbar_wait(bar_kwr, 0, a.err, abort_flag));
      if (ok2) {
        tc_fence_after();
        constexpr uint32_t idesc = make_idesc_bf16(128, kN, 0, 1);
#pragma unroll
        for (int ks = 0; ks < BPAD / 16; ++ks) {
          const uint64_t da = make_sdesc(base + kOffP + ks * 32, 16, 8 * Lay::kRowB, Lay::kPLayout);
          const uint64_t db =
              make_sdesc(base + Lay::kOffV + ks * 2048, BPAD * 128, 1024, kLayoutSW128);
          mma_bf16_ss(t_d, da, db, idesc, ks > 0 ? 1u : 0u);
        }
      }
    }

    // the phi(Q) S products: issued right after P V unless (shared
    // denominator) a row of the tile has to scale its phi(q) first, in which
    // case they follow the row owners' shared-denominator work (bar_a2)
    bool rescale = false;
    if (SHARED && !EARLY && tid == 128 && ok2) rescale = *rescale_flag != 0;
    auto issue_products = [&]() {
      if (ok2) ok2 = mbar_wait(SHARED && rescale ? bar_a2 : bar_a, 0, a.err, abort_flag);
      for (int c = 0; c < 4 && ok2; ++c) {
        ok2 = mbar_wait(bar_s + 8 * c, 0, a.err, abort_flag);
        if (!ok2) break;
        tc_fence_after();
        constexpr uint32_t idesc = make_idesc_tf32(128, kN, 0, 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // state rows 32c + 8kk .. +7 of every 32-column box: two 4-row
          // atoms of the 32-byte-chunk swizzle (MN-major tf32 layout)
          const uint64_t db = make_sdesc(base + kOffS + c * kChunkS + kk * 1024, 4096, 512,
                                         kLayoutSW128_32B);
          mma_tf32_ts(t_d, t_a + 32 * c + 8 * kk, db, idesc, 1u);
        }
      }
      if (ok2) mma_commit(bar_done);
    };
    if (!REUSE && !EARLY && tid == 128 && !rescale) issue_products();

    if (SHARED) {
      // phi(q) . z from warps 0-3; the output's 1 / denominator, and for rows
      // past the shift bound the factor e^{-m_s} into their phi(q)
      const bool oka = warp_all(ok && mbar_wait(bar_qz, 0, a.err, abort_flag));
      tc_fence_after();
      if (oka) {
        const float qz = ld_shared_f32(base + kOffQ + r * 128);
        if (m2 > kSharedShiftLog2) {
          ascale = exp2f(-m2);
          beta = 1.f / (lsum + ascale * qz);
        } else {
          beta = 1.f / (pscale * lsum + qz);
        }
        if (__any_sync(0xffffffffu, ascale != 1.f)) scale_tmem_row(t_a + lane_base, ascale);
        // the row's 1 / denominator for warps 0-3 (the other column half),
        // beside phi(q) . z in the row's bytes of the consumed Q tile
        if (!HALF) st_shared_f32(base + kOffQ + r * 128 + 4, beta);
      }
      tc_fence_before();
      mbar_arrive(bar_a2);
    }

    if (REUSE && tid == 128) {
      if (ok2) mma_commit(bar_done);   // P V is the whole product
    } else if (tid == 128) {
      if (rescale) issue_products();
      if (COMMIT && ok2) {
        // phi(K)^T V over the block's tokens into the columns phi(Q) used,
        // once the products that read them are complete
        ok2 = mbar_wait(bar_done, 0, a.err, abort_flag) && mbar_wait(bar_phik, 0, a.err, abort_flag);
        if (ok2) {
          tc_fence_after();
          // A = phi(K)^T: MN-major phi(K) in place, or K-major rows of the
          // projected map's features
          constexpr uint32_t idesc = make_idesc_bf16(128, kN, PROJ ? 0 : 1, 1);
#pragma unroll
          for (int ks = 0; ks < BPAD / 16; ++ks) {
            const uint64_t da =
                PROJ ? make_sdesc(base + kOffK + ks * 32, 16, 16 * BPAD,
                                  kmajor_layout<2 * BPAD>())
                     : make_sdesc(base + kOffK + ks * 2048, BPAD * 128, 1024, kLayoutSW128);
            const uint64_t db =
                make_sdesc(base + Lay::kOffV + ks * 2048, BPAD * 128, 1024, kLayoutSW128);
            mma_bf16_ss(t_a, da, db, idesc, ks > 0 ? 1u : 0u);
          }
          mma_commit(bar_ds);
        }
      }
    }
  }

  // ---- epilogue: all 8 warps; warp w: rows 32(w%4).., 64-column half w/4
  const int r = (warp & 3) * 32 + lane;
  const int hb = warp >> 2;
  const bool okd = warp_all(mbar_wait(bar_done, 0, a.err, abort_flag));
  tc_fence_after();
  if (SHARED && !HALF) {
    // warps 0-3 take their rows' 1 / denominator from the row owners (bar_a2:
    // the row owners are done with the Q tile's half these warps overwrite);
    // each column half then finishes on its own
    if (warp < 4) {
      const bool okb = warp_all(mbar_wait(bar_a2, 0, a.err, abort_flag));
      beta = okb ? ld_shared_f32(base + kOffQ + r * 128 + 4) : 1.f;
    }
  } else if (SHARED) {
    // column halves: both halves share each row's swizzled staging bytes, so
    // the row scales go through the (consumed) V tile and a CTA barrier
    float* rs = reinterpret_cast<float*>(smem_raw + (base - raw) + Lay::kOffV);
    if (warp >= 4) rs[r] = beta;
    named_barrier_sync(1, kThreads);
    beta = rs[r];
  }
  bool oko = true;
  if (REUSE) {
    // the merge weights likewise, and this warp's rows of O_pre in place
    float* rs = reinterpret_cast<float*>(smem_raw + (base - raw) + Lay::kOffV);
    if (warp >= 4) {
      rs[r] = ralpha;
      rs[kMT + r] = rbeta;
    }
    named_barrier_sync(1, kThreads);
    ralpha = rs[r];
    rbeta = rs[kMT + r];
    oko = warp_all(mbar_wait(bar_s + 8 * (warp & 3), 0, a.err, abort_flag));
  }
  // reuse: y = a D + b O_pre for the 32 columns of D in `acc` whose first
  // column is the start of 32 x 32 box `box` of the O_pre tile (row r)
  auto blend = [&](float (&acc)[32], uint32_t box) {
    const uint32_t ob = box + (r & 31) * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 lo = ld_shared_f4(ob + ((j ^ (r & 3)) << 5));
      const float4 hi = ld_shared_f4(ob + ((j ^ (r & 3)) << 5) + 16);
      const float o[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[8 * j + q] = fmaf(ralpha, acc[8 * j + q], rbeta * o[q]);
    }
  };
  if (HALF) {
    // warp w: rows 32(w%4).., columns 32(w/4).. of the CTA's 64; one SW128
    // box in the (consumed) Q region, one TMA store
    if (okd && oko) {
      const uint32_t row = base + kOffQ + r * 128;
      float acc[32];
      tmem_ld32_sync(t_d + lane_base + hb * 32, acc);
      if (REUSE) blend(acc, base + kOffS + (r >> 5) * kChunkS + hb * 4096);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = hb * 4 + q;
        const float* e = acc + 8 * q;
        st_shared_v4(row + ((j ^ (r & 7)) << 4), pack_bf16x2(e[0] * beta, e[1] * beta),
                     pack_bf16x2(e[2] * beta, e[3] * beta),
                     pack_bf16x2(e[4] * beta, e[5] * beta),
                     pack_bf16x2(e[6] * beta, e[7] * beta));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_barrier_sync(2, kThreads);
    if (tid == 0 && !*abort_flag) {
      tma_store_3d(&tmY, base + kOffQ, 64 * half, mt * kMT, u);
      bulk_commit_group();
    }
  } else {
  if (okd && oko) {
    // bf16 tile of this 64-column half -> the (consumed) Q region, SW128
    const uint32_t row = base + kOffQ + hb * 16384 + r * 128;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float acc[32];
      tmem_ld32_sync(t_d + lane_base + hb * 64 + cc * 32, acc);
      if (REUSE) blend(acc, base + kOffS + (r >> 5) * kChunkS + (hb * 2 + cc) * 4096);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = cc * 4 + q;
        const float* e = acc + 8 * q;
        st_shared_v4(row + ((j ^ (r & 7)) << 4), pack_bf16x2(e[0] * beta, e[1] * beta),
                     pack_bf16x2(e[2] * beta, e[3] * beta),
                     pack_bf16x2(e[4] * beta, e[5] * beta),
                     pack_bf16x2(e[6] * beta, e[7] * beta));
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  named_barrier_sync(2 + hb, 128);
  if ((tid & 127) == 0 && !*abort_flag) {
    tma_store_3d(&tmY, base + kOffQ + hb * 16384, 64 * hb, mt * kMT, u);
    bulk_commit_group();
  }
  }
  if (COMMIT) {
    // phi(K)^T V over the consumed state tile (32-byte-chunk swizzle: chunk
    // j of row rr of a 32 x 32 box sits at j ^ (rr % 4)), then S += it by
    // TMA reduce-add (the add is done at L2)
    const bool okc = warp_all(mbar_wait(bar_ds, 0, a.err, abort_flag));
    tc_fence_after();
    if (okc) {
      const int rr = r & 31;
      const uint32_t rowb = base + kOffS + (r >> 5) * kChunkS + rr * 128;
      // warp w: columns (kN / 2) (w / 4).. of the CTA's dS, 32 at a time
#pragma unroll
      for (int cc = 0; cc < kN / 64; ++cc) {
        float dsv[32];
        tmem_ld32_sync(t_a + lane_base + hb * (kN / 2) + cc * 32, dsv);
        const uint32_t box = rowb + (hb * (kN / 64) + cc) * 4096;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t addr = box + ((j ^ (rr & 3)) << 5);
          st_shared_f4(addr, make_float4(dsv[8 * j], dsv[8 * j + 1], dsv[8 * j + 2],
                                         dsv[8 * j + 3]));
          st_shared_f4(addr + 16, make_float4(dsv[8 * j + 4], dsv[8 * j + 5], dsv[8 * j + 6],
                                              dsv[8 * j + 7]));
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && okc && !*abort_flag) {
      for (int c = 0; c < 4; ++c)
        for (int nn = 0; nn < kN / 32; ++nn)
          tma_reduce_add_3d(&tmS, base + kOffS + c * kChunkS + nn * 4096,
                            32 * (HALF ? 2 * half + nn : nn), 32 * c, u);
      bulk_commit_group();
    }
  }
  // every TMEM read is done once both halves passed their barrier
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if ((tid & 127) == 0) bulk_wait_group_read0();   // shared memory stays until read
}

template <int BPAD, bool SHARED, bool COMMIT, int FMAP, bool HALF = false, bool REUSE = false>
int launch_cfg(const Ctx& c, const CUtensorMap (&tm)[6], const StepArgs& a, int grid) {
  using Lay = StepLayout<BPAD>;
  auto kern = k_step_bf16<BPAD, SHARED, COMMIT, FMAP, HALF, REUSE>;
  static Prepared prepared;
  if (!prepare_kernel(c, kern, (int)Lay::kSmem, prepared)) return -5;
  return launch_pdl(kern, (HALF ? 2 : 1) * grid, kThreads, Lay::kSmem, c.stream, tm[0], tm[1],
                    tm[2], tm[3], tm[4], tm[5], a);
}

// Column halves when the grid would fill at most one CTA per SM (and the
// map is elementwise).
template <int BPAD, int FMAP>
int launch_fmap(const Ctx& c, const CUtensorMap (&tm)[6], const StepArgs& a, int grid, int shared,
                int commit) {
  const bool halves = FMAP != kFmapReluProj && grid <= c.sm_count;
  if (commit)
    return halves ? launch_cfg<BPAD, false, true, FMAP, FMAP != kFmapReluProj>(c, tm, a, grid)
                  : launch_cfg<BPAD, false, true, FMAP>(c, tm, a, grid);
  if (halves)
    return shared ? launch_cfg<BPAD, true, false, FMAP, FMAP != kFmapReluProj>(c, tm, a, grid)
                  : launch_cfg<BPAD, false, false, FMAP, FMAP != kFmapReluProj>(c, tm, a, grid);
  return shared ? launch_cfg<BPAD, true, false, FMAP>(c, tm, a, grid)
                : launch_cfg<BPAD, false, false, FMAP>(c, tm, a, grid);
}

template <int BPAD>
int launch_bpad(const Ctx& c, const CUtensorMap (&tm)[6], const StepArgs& a, int grid, int shared,
                int commit, int fmap) {
  switch (fmap) {
    case kFmapRelu: return launch_fmap<BPAD, kFmapRelu>(c, tm, a, grid, shared, commit);
    case kFmapElu1: return launch_fmap<BPAD, kFmapElu1>(c, tm, a, grid, shared, commit);
    default: return launch_fmap<BPAD, kFmapReluProj>(c, tm, a, grid, shared, commit);
  }
}

}  // namespace

int launch_step_bf16(const Ctx& c, const void* Q, const void* K, const void* V, const float* S,
                     const float* z, void* Y, int n, int hq, int hkv, int b, float scale,
                     int shared, int fmap, const void* W, float* commit_z, int commit) {
  const int G = hq / hkv;
  const int rows = G * b;
  const int units = n * hkv;
  const int bpad = b <= 16 ? 16 : (b <= 32 ? 32 : 64);
  const int mtiles = (rows + kMT - 1) / kMT;

  // tm: Q, K, V, S, Y, W (Q's map stands in for W under the elementwise maps)
  CUtensorMap tm[6];
  const uint64_t dq[3] = {(uint64_t)kD, (uint64_t)rows, (uint64_t)units};
  const uint64_t sq[2] = {kD * 2ull, (uint64_t)rows * kD * 2ull};
  const uint32_t bq[3] = {64, kMT, 1};
  const uint64_t dk[3] = {(uint64_t)kD, (uint64_t)b, (uint64_t)units};
  const uint64_t sk[2] = {kD * 2ull, (uint64_t)b * kD * 2ull};
  const uint32_t bk[3] = {64, (uint32_t)bpad, 1};
  const uint64_t ds[3] = {(uint64_t)kD, (uint64_t)kD, (uint64_t)units};
  const uint64_t ss[2] = {kD * 4ull, (uint64_t)kD * kD * 4ull};
  const uint32_t bs[3] = {32, 32, 1};
  const uint64_t dw[3] = {(uint64_t)kD, (uint64_t)kD, (uint64_t)hkv};
  const uint64_t sw[2] = {kD * 2ull, (uint64_t)kD * kD * 2ull};
  const uint32_t bw[3] = {64, (uint32_t)kD, 1};
  if (!encode_tmap(&tm[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Q, dq, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tm[4], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Y, dq, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tm[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, K, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tm[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tm[3], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, S, ds, ss, bs,
                   CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B))
    return -5;
  if (fmap == kFmapReluProj) {
    if (!encode_tmap(&tm[5], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, W, dw, sw, bw,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return -5;
  } else {
    tm[5] = tm[0];
  }

  StepArgs a;
  a.z = z;
  a.lpre = nullptr;
  a.zc = commit ? commit_z : nullptr;
  a.err = c.dev_err;
  a.hkv = hkv;
  a.rows = rows;
  a.b = b;
  a.mtiles = mtiles;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  const int grid = units * mtiles;
  switch (bpad) {
    case 16: return launch_bpad<16>(c, tm, a, grid, shared, commit, fmap);
    case 32: return launch_bpad<32>(c, tm, a, grid, shared, commit, fmap);
    default: return launch_bpad<64>(c, tm, a, grid, shared, commit, fmap);
  }
}

// The reuse path's block pass: every query row's attention over the active
// block, merged with its cached prefix part (O_pre [units][rows][128] fp32,
// L_pre [units][rows] natural-log normalisers; rows = G * b).
int launch_reuse_block_bf16(const Ctx& c, const void* Q, const void* K, const void* V,
                            const float* O_pre, const float* L_pre, void* Y, int n, int hq,
                            int hkv, int b, float scale) {
  const int G = hq / hkv;
  const int rows = G * b;
  const int units = n * hkv;
  const int bpad = b <= 16 ? 16 : (b <= 32 ? 32 : 64);
  const int mtiles = (rows + kMT - 1) / kMT;
  CUtensorMap tm[6];
  const uint64_t dq[3] = {(uint64_t)kD, (uint64_t)rows, (uint64_t)units};
  const uint64_t sq[2] = {kD * 2ull, (uint64_t)rows * kD * 2ull};
  const uint32_t bq[3] = {64, kMT, 1};
  const uint64_t dk[3] = {(uint64_t)kD, (uint64_t)b, (uint64_t)units};
  const uint64_t sk[2] = {kD * 2ull, (uint64_t)b * kD * 2ull};
  const uint32_t bk[3] = {64, (uint32_t)bpad, 1};
  const uint64_t dob[3] = {(uint64_t)kD, (uint64_t)rows, (uint64_t)units};
  const uint64_t sob[2] = {kD * 4ull, (uint64_t)rows * kD * 4ull};
  const uint32_t bob[3] = {32, 32, 1};
  if (!encode_tmap(&tm[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Q, dq, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tm[4], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Y, dq, sq, bq,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tm[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, K, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tm[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, V, dk, sk, bk,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap(&tm[3], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, O_pre, dob, sob, bob,
                   CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B))
    return -5;
  tm[5] = tm[0];
  StepArgs a;
  a.z = nullptr;
  a.lpre = L_pre;
  a.zc = nullptr;
  a.err = c.dev_err;
  a.hkv = hkv;
  a.rows = rows;
  a.b = b;
  a.mtiles = mtiles;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  const int grid = units * mtiles;
  const bool halves = grid <= c.sm_count;
  switch (bpad) {
    case 16:
      return halves ? launch_cfg<16, false, false, kFmapRelu, true, true>(c, tm, a, grid)
                    : launch_cfg<16, false, false, kFmapRelu, false, true>(c, tm, a, grid);
    case 32:
      return halves ? launch_cfg<32, false, false, kFmapRelu, true, true>(c, tm, a, grid)
                    : launch_cfg<32, false, false, kFmapRelu, false, true>(c, tm, a, grid);
    default:
      return halves ? launch_cfg<64, false, false, kFmapRelu, true, true>(c, tm, a, grid)
                    : launch_cfg<64, false, false, kFmapRelu, false, true>(c, tm, a, grid);
  }
}

}  // namespace bha
