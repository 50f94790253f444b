/*
 * bha.h -- C ABI of block-hybrid attention on NVIDIA B200 (sm_100a).
 *
 * Method: "Retrofitting Linear Attention into Diffusion Language Models"
 * (Kim, Roh, Kim; arXiv 2608.06628).  The paper-daily summary page gives the
 * core formula (section 核心公式与算法) and a worked example (section
 * 具体技术细节示例); the fugumt page carries the abstract.  During blockwise
 * semi-autoregressive decoding, attention inside the active denoising block
 * is exact softmax, and attention over all previous blocks is linear
 * attention through a per-KV-head prefix state:
 *
 *     y   = softmax(Q_a K_a^T * scale) V_a + phi(Q_a) S_p
 *     S_p = sum over committed tokens t of phi(k_t)^T v_t      (d x d)
 *     phi = ReLU (elementwise; the worked example's kernel feature map)
 *
 * Tensors and layouts (row-major, contiguous, device memory):
 *   Q_a, Y      [n][hq][b][d]         active-block queries / outputs
 *   K_a, V_a    [n][hkv][b][d]        active-block keys / values
 *   K_p, V_p    [n][hkv][T][d]        prompt keys / values (prefill)
 *   K_c, V_c    [n][hkv][cap][d]      KV cache, first P tokens valid
 *   S           [n][hkv][d][d] fp32   S[r][c] = sum_t phi(k_t)[r] v_t[c]
 *   z           [n][hkv][d]    fp32   z[r]    = sum_t phi(k_t)[r]
 * GQA: query head h reads KV head h / (hq / hkv) (contiguous grouping).
 * Element type of Q/K/V/Y: bha_dtype (bf16, or fp32 for the reference mode);
 * S and z are always fp32, and every path accumulates in fp32.
 *
 * Ownership: the caller allocates and owns every buffer, the workspace and
 * the stream.  No call allocates memory.  The library's device code holds
 * one 4-byte word per GPU that records a kernel-side error (read with
 * bha_device_error) and the fixed 32 MiB array of bha_state_prefill_noalloc
 * (below); both exist wherever the CUDA runtime has loaded the library's
 * device code into a context.  Under lazy module loading (the default) that
 * is the first call on a device; under eager loading
 * (CUDA_MODULE_LOADING=EAGER) every context holds both from its creation,
 * the 32 MiB included, whether or not bha_state_prefill_noalloc is called.
 * The host side caches each device's symbol addresses per CUDA context and
 * looks them up again after cudaDeviceReset has replaced the context.
 *
 * Behaviour: every compute call validates its arguments before any launch,
 * returns a negative bha_status on failure (nothing launched), otherwise
 * enqueues its kernels on `stream` and returns BHA_OK without waiting.  A
 * launch failure reported by the runtime returns BHA_ERR_CUDA.  Kernels wait
 * on their own asynchronous copies with a bounded spin; if a wait runs out
 * they record BHA_ERR_TIMEOUT in the device error word and return.  The
 * outputs of that call, and the state S, z of a call that updates them in
 * place, are then undefined.
 * Pointers must be 16-byte aligned (BHA_ERR_MISALIGNED).  Outputs must not
 * overlap inputs (BHA_ERR_INVALID_ARG).  n = 0 is a valid empty call.
 *
 * Supported shapes (else BHA_ERR_UNSUPPORTED):
 *   BHA_BF16: d == 128, 1 <= b <= 64 (tensor-core paths, sm_100a).
 *   BHA_F32 : 1 <= d <= 128, d % 4 == 0, 1 <= b <= 64 (CUDA-core reference
 *             mode, used for the worked example and 1e-4 checks).
 */
#ifndef BHA_H
#define BHA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream; identical to cudaStream_t (NULL = legacy default stream). */
typedef struct CUstream_st *bha_stream_t;

typedef enum {
    BHA_OK = 0,
    BHA_ERR_INVALID_ARG = -1, /* null pointer, bad count, aliasing, hq % hkv */
    BHA_ERR_UNSUPPORTED = -2, /* shape/dtype outside the supported sets     */
    BHA_ERR_MISALIGNED = -3,  /* a pointer is not 16-byte aligned           */
    BHA_ERR_WORKSPACE = -4,   /* workspace NULL or smaller than required    */
    BHA_ERR_CUDA = -5,        /* the CUDA runtime reported an error         */
    BHA_ERR_TIMEOUT = -6,     /* a kernel's bounded wait ran out            */
    BHA_ERR_DEVICE = -7       /* a kernel detected an internal fault        */
} bha_status;

typedef enum { BHA_BF16 = 0, BHA_F32 = 1 } bha_dtype;

/* Normalise the two terms by one shared denominator (an engineer-added
 * option; the pages add the terms unnormalised):
 *   y = (sum_j e^{s_j - m} v_j + e^{-m} phi(q) S) /
 *       (sum_j e^{s_j - m}     + e^{-m} phi(q) . z),   m = max_j s_j.
 * Requires z.  The pages have no counterpart of this option. */
#define BHA_FLAG_SHARED_DENOM 1u

/* Human-readable name of a bha_status value (never NULL). */
const char *bha_status_string(int status);

/* ABI version, currently 1. */
int bha_version(void);

/*
 * Prefill: fold a prompt into the prefix state (the prompt counts as the
 * "previous blocks" of the first generated block; follows from the abstract's
 * linear attention over previous blocks and the worked example's S_1).
 *   S = phi(K_p)^T V_p,  z = sum_t phi(k_t)        (overwrites S and z)
 * K, V: [n][hkv][T][d]; S: [n][hkv][d][d]; z: [n][hkv][d] or NULL.
 * T = 0 writes S = 0 (and z = 0).  The bf16 path splits T into chunks
 * reduced in a fixed order through `workspace` (deterministic result);
 * workspace may be NULL when bha_state_prefill_workspace_size returns 0.
 */
size_t bha_state_prefill_workspace_size(int n, int hkv, int T, int d,
                                        bha_dtype dtype);
int bha_state_prefill(const void *K, const void *V, int n, int hkv, int T,
                      int d, bha_dtype dtype, float *S, float *z,
                      void *workspace, size_t workspace_bytes,
                      bha_stream_t stream);

/*
 * Allocation-free variant of bha_state_prefill (the paper has no counterpart:
 * this is an interface for callers that cannot allocate device memory, such
 * as plugins inside a host application that owns all device memory or
 * runtimes that forbid allocation once serving has started).  Same
 * arguments and result as bha_state_prefill without the workspace: the
 * chunk partials go to a 32 MiB array held in the library's device memory
 * on every GPU that uses it, until the process exits.  Returns
 * BHA_ERR_WORKSPACE, launching nothing, when bha_state_prefill_workspace_size
 * exceeds 32 MiB.  The array's device address is looked up on the first
 * call made in each CUDA context: the first call on a device, and the first
 * after cudaDeviceReset (make that call before any stream capture).  All
 * calls on a device share the array: calls whose kernels overlap on the GPU
 * race on it.  It holds nothing that must start at zero.  Where the array is
 * reserved depends on module loading: see Ownership above.
 */
int bha_state_prefill_noalloc(const void *K, const void *V, int n, int hkv,
                              int T, int d, bha_dtype dtype, float *S,
                              float *z, bha_stream_t stream);

/*
 * Commit: add a finalised block to the prefix state (worked example:
 * S_{1,2} = phi(K_1)^T V_1 + phi(K_2)^T V_2).
 *   S += phi(K_blk)^T V_blk,  z += sum_t phi(k_t)     (in place)
 * Kb, Vb: [n][hkv][b][d]; S: [n][hkv][d][d]; z: [n][hkv][d] or NULL.
 */
int bha_state_commit(const void *Kb, const void *Vb, int n, int hkv, int b,
                     int d, bha_dtype dtype, float *S, float *z,
                     bha_stream_t stream);

/*
 * One denoising step of block-hybrid attention (core formula): for every
 * query row i of the active block,
 *   y_i = sum_j softmax_j(scale q_i . k_j) v_j  +  phi(q_i) S
 * with j over the b block tokens (bidirectional, no mask) and S the state
 * of all previous blocks.  scale <= 0 selects 1/sqrt(d).  flags:
 * BHA_FLAG_SHARED_DENOM (needs z).  Y must not overlap any input.
 */
int bha_hybrid_step(const void *Qa, const void *Ka, const void *Va,
                    const float *S, const float *z, void *Y, int n, int hq,
                    int hkv, int b, int d, float scale, unsigned flags,
                    bha_dtype dtype, bha_stream_t stream);

/*
 * The block's last denoising step fused with its commit: the result of
 * bha_hybrid_step on (Qa, Ka, Va, S, z), after which S += phi(Ka)^T Va and
 * z += sum_t phi(ka_t) (z may be NULL in the default mode) -- the two steps
 * the worked example takes when a block is finalised (block 2 uses S_1, then
 * S_{1,2} = S_1 + phi(K_2)^T V_2).  In the default mode with G * b <= 128
 * this is one kernel that reads the state once; otherwise it launches the
 * step and the commit kernels back to back.  Y must not overlap any input,
 * S or z; S and z must not overlap the inputs.  If a kernel of this call
 * records BHA_ERR_TIMEOUT (bha_device_error), the contents of S and z are
 * undefined afterwards: the update is not atomic per (request, KV head) --
 * on small grids two CTAs each add half of the columns -- so rebuild the
 * state (for example by a prefill) before using it again.
 */
int bha_hybrid_step_commit(const void *Qa, const void *Ka, const void *Va,
                           float *S, float *z, void *Y, int n, int hq,
                           int hkv, int b, int d, float scale, unsigned flags,
                           bha_dtype dtype, bha_stream_t stream);

/*
 * Comparison path: exact softmax attention of the active block over the
 * whole KV cache plus the block itself (the abstract's baseline, where
 * every denoising step attends to all previous blocks):
 *   y_i = sum_j softmax_j(scale q_i . k_j) v_j,  j in [K_c[0:P] || K_a]
 * Kc, Vc: [n][hkv][cap][d] with P <= cap valid tokens.  The bf16 path splits
 * the P + b keys into chunks merged by log-sum-exp through `workspace`.
 */
size_t bha_prefix_softmax_workspace_size(int n, int hq, int hkv, int b,
                                         int d, int P, bha_dtype dtype);
int bha_prefix_softmax(const void *Qa, const void *Kc, const void *Vc, int P,
                       int cap, const void *Ka, const void *Va, void *Y,
                       int n, int hq, int hkv, int b, int d, float scale,
                       bha_dtype dtype, void *workspace,
                       size_t workspace_bytes, bha_stream_t stream);

/*
 * Feature maps.  The method-details section (技术方法详解) of the paper-daily
 * summary page has the previous blocks go through a kernel-function
 * approximation, and its future-work section (未来研究方向) names better
 * kernel functions as the next step; the worked example uses ReLU.  Every
 * call above uses BHA_FMAP_RELU.  The _fm variants below take the map:
 *   BHA_FMAP_RELU       phi(x)_j = max(x_j, 0)
 *   BHA_FMAP_ELU1       phi(x)_j = x_j + 1 if x_j > 0, else exp(x_j)
 *   BHA_FMAP_RELU_PROJ  phi(x)_j = max(sum_i x_i W[g][i][j], 0)
 * W: [hkv][d][d], row-major, element type = dtype; KV head g's queries and
 * keys use W[g] (queries by the GQA map), so phi keeps d features and S
 * stays d x d.  W must be non-NULL and 16-byte aligned for
 * BHA_FMAP_RELU_PROJ and NULL otherwise (BHA_ERR_INVALID_ARG), and must not
 * overlap an output.  The bf16 path evaluates elu + 1 in packed bf16
 * arithmetic and rounds ReLU(x W_g) of keys to bf16 (phi(k) is a bf16 tensor-
 * core operand, as in a bf16 model); phi(q) enters the phi(q) S product as
 * tf32, like S.
 */
typedef enum {
    BHA_FMAP_RELU = 0,
    BHA_FMAP_ELU1 = 1,
    BHA_FMAP_RELU_PROJ = 2
} bha_fmap;

/* bha_state_prefill with feature map `fmap` (workspace as for
 * bha_state_prefill: the size does not depend on the map). */
int bha_state_prefill_fm(const void *K, const void *V, int n, int hkv, int T,
                         int d, bha_dtype dtype, bha_fmap fmap, const void *W,
                         float *S, float *z, void *workspace,
                         size_t workspace_bytes, bha_stream_t stream);

/* bha_state_commit with feature map `fmap`. */
int bha_state_commit_fm(const void *Kb, const void *Vb, int n, int hkv, int b,
                        int d, bha_dtype dtype, bha_fmap fmap, const void *W,
                        float *S, float *z, bha_stream_t stream);

/* bha_hybrid_step with feature map `fmap` (phi of the queries; S and z
 * must have been built with the same map). */
int bha_hybrid_step_fm(const void *Qa, const void *Ka, const void *Va,
                       const float *S, const float *z, void *Y, int n, int hq,
                       int hkv, int b, int d, float scale, unsigned flags,
                       bha_dtype dtype, bha_fmap fmap, const void *W,
                       bha_stream_t stream);

/* bha_hybrid_step_commit with feature map `fmap` (one kernel in the same
 * cases as bha_hybrid_step_commit, for every map). */
int bha_hybrid_step_commit_fm(const void *Qa, const void *Ka, const void *Va,
                              float *S, float *z, void *Y, int n, int hq,
                              int hkv, int b, int d, float scale,
                              unsigned flags, bha_dtype dtype, bha_fmap fmap,
                              const void *W, bha_stream_t stream);

/*
 * Ragged and paged batches.  The method-details section (技术方法详解) of the
 * summary page pairs the method with KV-cache management and its related
 * work (相关工作) names PagedAttention: requests of one batch carry caches
 * and prompts of their own lengths.
 */

/*
 * Exact path over a paged KV cache with per-request cache lengths: for each
 * request i, the result of bha_prefix_softmax with its own cache, its first
 * P_lens[i] tokens, token t at row t % page_size of page
 * block_table[i][t / page_size].
 *   Kpool, Vpool  [num_pages][hkv][page_size][d]   pages of keys / values
 *   block_table   [n][max_pages] int32, device memory
 *   P_lens        [n] int32, device memory; clamped to [0, max_pages * page_size]
 * page_size is a power of two from 16 to 256 (else BHA_ERR_UNSUPPORTED).
 * Pool slots past a request's cache may hold anything; a page number outside
 * [0, num_pages) reads as zero rows.  block_table and P_lens must be 4-byte
 * aligned.  The workspace is sized for the longest cache,
 * max_pages * page_size tokens.
 */
size_t bha_prefix_softmax_paged_workspace_size(int n, int hq, int hkv, int b,
                                               int d, int max_pages,
                                               int page_size, bha_dtype dtype);
int bha_prefix_softmax_paged(const void *Qa, const void *Kpool,
                             const void *Vpool, int num_pages, int page_size,
                             const int *block_table, int max_pages,
                             const int *P_lens, const void *Ka,
                             const void *Va, void *Y, int n, int hq, int hkv,
                             int b, int d, float scale, bha_dtype dtype,
                             void *workspace, size_t workspace_bytes,
                             bha_stream_t stream);

/*
 * Prefill of prompts of different lengths: request i folds its first
 * T_lens[i] tokens of K, V [n][hkv][Tmax][d] (T_lens: [n] int32 in device
 * memory, 4-byte aligned, clamped to [0, Tmax]); rows past T_lens[i] are
 * padding and may hold anything.  Overwrites S and z as bha_state_prefill
 * does; feature map as for the _fm calls; the workspace is that of
 * bha_state_prefill for Tmax tokens.
 */
int bha_state_prefill_ragged(const void *K, const void *V, const int *T_lens,
                             int n, int hkv, int Tmax, int d, bha_dtype dtype,
                             bha_fmap fmap, const void *W, float *S, float *z,
                             void *workspace, size_t workspace_bytes,
                             bha_stream_t stream);

/*
 * Reuse of prefix attention for stable tokens (the LoSA page: gist.science
 * explainer of arXiv 2604.12056, section "3. 方法论 LoSA" -- 局部性剪枝
 * locality pruning, 缓存复用 cache reuse, 初始化策略 initialisation -- and
 * "技术细节" technical details), applied to the exact comparison path with a
 * dense prefix pass over the active tokens (the page's sparse selector is not
 * part of this library).  One denoising step of a block:
 *   1. score_i = mean over every query head h and dimension c of
 *      (Qa[n][h][i][c] - Qprev[n][h][i][c])^2, the MSE of token i's query
 *      since the previous denoising step (evaluated in fp64: per head the
 *      squares summed in column order, then the heads summed in order, so
 *      the selection is reproducible bit for bit);
 *   2. the active set of request n: the k tokens with the largest score,
 *      ties to the lower token index;
 *   3. for an active token, every query head's softmax attention over the
 *      cache alone, as its normalised output and natural-log normaliser
 *      lse_p = log sum_{j<P} exp(scale q . k_j), replaces the token's entries
 *      of the reuse cache (O_pre, L_pre); a stable token keeps the entries
 *      the previous step left (computed with an earlier query);
 *   4. y = (e^{lse_p - M} o_p + e^{lse_b - M} o_b) / (e^{lse_p - M} + e^{lse_b - M}),
 *      M = max(lse_p, lse_b), with o_b, lse_b the token's softmax attention
 *      over the b block tokens with its current query (P = 0: y = o_b).
 * Qprev == NULL (the block's first denoising step, the page's dense
 * initialisation) or k >= b makes every token active; the result is then
 * that of bha_prefix_softmax.  k = 0 makes every token stable.
 *   Qa, Qprev     [n][hq][b][d]     this and the previous step's queries
 *   O_pre         [n][hq][b][d] fp32, L_pre [n][hq][b] fp32: the reuse
 *                 cache, b x (d + 1) values per query head, read for stable
 *                 tokens and written for active ones; it must come from the
 *                 previous step of the same block (any contents when every
 *                 token is active)
 *   active        [n][k] int32 or NULL: the active tokens of each request in
 *                 increasing order, written on steps that select (Qprev set,
 *                 0 < k < b), untouched otherwise
 * Other arguments as for bha_prefix_softmax, and hq * b <= 8192 (else
 * BHA_ERR_UNSUPPORTED).  BHA_F32 is the CUDA-core reference mode (one CTA
 * per query row; no workspace).  The workspace size covers both kinds of step (first
 * and later) for the given k.  Y must not overlap any input or the cache;
 * O_pre, L_pre and active must not overlap the inputs or each other.
 */
size_t bha_prefix_softmax_reuse_workspace_size(int n, int hq, int hkv, int b,
                                               int d, int P, int k,
                                               bha_dtype dtype);
int bha_prefix_softmax_reuse(const void *Qa, const void *Qprev,
                             const void *Kc, const void *Vc, int P, int cap,
                             const void *Ka, const void *Va, void *Y,
                             float *O_pre, float *L_pre, int *active, int k,
                             int n, int hq, int hkv, int b, int d, float scale,
                             bha_dtype dtype, void *workspace,
                             size_t workspace_bytes, bha_stream_t stream);

/*
 * Block partition of a length-L sequence into blocks of B tokens, the last
 * one possibly short (worked example: L=10, B=4 -> tokens 1-4, 5-8, 9-10).
 * Host-only.  Writes bounds[0..k] = {0, B, 2B, ..., L} and returns k, the
 * number of blocks; returns BHA_ERR_INVALID_ARG for L < 0, B < 1 or a NULL
 * bounds, BHA_ERR_WORKSPACE if max_bounds < k + 1.
 */
int bha_block_partition(int L, int B, int *bounds, int max_bounds);

/*
 * Synchronises the current device and returns the device error word
 * (BHA_OK, BHA_ERR_TIMEOUT or BHA_ERR_DEVICE) recorded by any kernel since
 * the last reset; reset != 0 clears it.  Returns BHA_ERR_CUDA if the device
 * cannot be read.
 */
int bha_device_error(int reset);

/*
 * Self-test of the timeout path (diagnostics; the pages have no counterpart):
 * launches one small kernel that waits on a barrier nothing will complete,
 * with a 10 ms limit instead of the kernels' 1 s.  The wait gives up, the
 * kernel records BHA_ERR_TIMEOUT in the device error word and exits normally,
 * so the context stays usable.  Returns BHA_OK once launched.
 */
int bha_selftest_timeout(bha_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* BHA_H */
