/*
 * Plain fp64 CPU oracle for block-hybrid attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library and never calls it.
 *
 * Source of the method: "Retrofitting Linear Attention into Diffusion
 * Language Models" (Kim, Roh, Kim; arXiv 2608.06628) as summarised on the
 * paper-daily page (sections "核心公式与算法" = core formula and
 * "具体技术细节示例" = worked example) and the fugumt abstract page.
 *
 *   y = Softmax(Q_a K_a^T) V_a + phi(Q_a) S_p,   S_p = sum_t phi(k_t)^T v_t
 *
 * with phi = ReLU (worked example), the softmax scaled by 1/sqrt(d) and the
 * query feature term taken on the active block's queries (the worked example
 * writes phi(Q_2) S_1 for block 2).  Every routine here is written as the
 * plain definition, one output element at a time, in double precision; no
 * blocking, fusion or reordering beyond the definition.
 *
 * Layouts (all row-major, contiguous):
 *   Q, Y            [n][hq][b][d]
 *   K, V (block)    [n][hkv][b][d]
 *   K, V (prompt)   [units][T][d]           (units = n*hkv)
 *   K, V (cache)    [n][hkv][cap][d], the first P tokens valid
 *   S               [units][d][d]   S[r][c] = sum_t phi(k_t)[r] * v_t[c]
 *   z               [units][d]      z[r]    = sum_t phi(k_t)[r]
 * GQA: query head h reads KV head h / (hq/hkv) (contiguous grouping).
 *
 * parity pins: see tests/test_oracle_pins.py.  The shared-denominator
 * variant is not on the pages (an engineer-added option); it is pinned only
 * by its own reduction cases and a brute-force restatement over prefix
 * tokens, not by any page value.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double relu(double x) { return x > 0.0 ? x : 0.0; }

/*
 * Kernel feature maps phi.  The worked example (paper-daily summary page,
 * 具体技术细节示例) takes phi = ReLU; the method details (技术方法详解) speak of
 * kernel-function approximations in general and list better kernels as
 * future work (未来研究方向), so two more maps are provided:
 *   fmap 0  ReLU        phi(x)_c = max(x_c, 0)
 *   fmap 1  ELU + 1     phi(x)_c = x_c + 1 if x_c > 0 else exp(x_c)
 *   fmap 2  projected   phi(x)_c = max(sum_r x_r W[r][c], 0), W a d x d matrix
 * out[c] = phi(x)_c for one d-vector x; W is the KV head's projection
 * (ignored unless fmap = 2).
 */
static void phi_vec(const double *x, long d, int fmap, const double *W, double *out)
{
    for (long c = 0; c < d; ++c) {
        if (fmap == 2) {
            double acc = 0.0;
            for (long r = 0; r < d; ++r)
                acc += x[r] * W[r * d + c];
            out[c] = relu(acc);
        } else if (fmap == 1) {
            out[c] = x[c] > 0.0 ? x[c] + 1.0 : exp(x[c]);
        } else {
            out[c] = relu(x[c]);
        }
    }
}

static int g_threads = 1;

/* Number of OpenMP threads the routines below use (1 = single-threaded). */
int oracle_set_threads(int n)
{
    if (n < 1) n = 1;
    g_threads = n;
    return g_threads;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_num_procs();
#else
    return 1;
#endif
}

/*
 * Prefix state of a prompt (the prompt counts as "previous blocks"):
 *   S[u][r][c] = sum_{t<T} phi(K[u][t])[r] * V[u][t][c]
 *   z[u][r]    = sum_{t<T} phi(K[u][t])[r]
 * T = 0 gives S = 0, z = 0.  z may be NULL.  W holds w_units projections
 * (one per KV head); unit u uses W[u % w_units] (units are (n, kvh) pairs,
 * KV head fastest).  Worked example: S_1 = phi(K_1)^T V_1.
 */
void oracle_state_prefill(const double *K, const double *V, long units, long T,
                          long d, double *S, double *z, int fmap, const double *W,
                          long w_units)
{
    long u;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (u = 0; u < units; ++u) {
        const double *Ku = K + u * T * d;
        const double *Vu = V + u * T * d;
        const double *Wu = W ? W + (u % w_units) * d * d : NULL;
        double *Su = S + u * d * d;
        double *fk = (double *)malloc(sizeof(double) * (size_t)(T * d > 0 ? T * d : 1));
        for (long t = 0; t < T; ++t)
            phi_vec(Ku + t * d, d, fmap, Wu, fk + t * d);
        for (long r = 0; r < d; ++r) {
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long t = 0; t < T; ++t)
                    acc += fk[t * d + r] * Vu[t * d + c];
                Su[r * d + c] = acc;
            }
            if (z) {
                double zs = 0.0;
                for (long t = 0; t < T; ++t)
                    zs += fk[t * d + r];
                z[u * d + r] = zs;
            }
        }
        free(fk);
    }
}

/*
 * Block commit when a block is finalised:
 *   S[u] += phi(Kb[u])^T Vb[u],   z[u] += sum_t phi(Kb[u][t])
 * Worked example: S_{1,2} = phi(K_1)^T V_1 + phi(K_2)^T V_2.
 * Kb, Vb are [units][b][d].  z may be NULL.  W as for the prefill.
 */
void oracle_state_commit(double *S, double *z, const double *Kb,
                         const double *Vb, long units, long b, long d, int fmap,
                         const double *W, long w_units)
{
    long u;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (u = 0; u < units; ++u) {
        const double *Ku = Kb + u * b * d;
        const double *Vu = Vb + u * b * d;
        const double *Wu = W ? W + (u % w_units) * d * d : NULL;
        double *Su = S + u * d * d;
        double *fk = (double *)malloc(sizeof(double) * (size_t)(b * d));
        for (long t = 0; t < b; ++t)
            phi_vec(Ku + t * d, d, fmap, Wu, fk + t * d);
        for (long r = 0; r < d; ++r) {
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long t = 0; t < b; ++t)
                    acc += fk[t * d + r] * Vu[t * d + c];
                Su[r * d + c] += acc;
            }
            if (z) {
                double zs = 0.0;
                for (long t = 0; t < b; ++t)
                    zs += fk[t * d + r];
                z[u * d + r] += zs;
            }
        }
        free(fk);
    }
}

/*
 * One denoising step of block-hybrid attention for every query row of the
 * active block (core formula; worked example, blocks 2 and 3).
 *
 * For request n, query head h (KV head g = h / (hq/hkv)), query row i:
 *   s_j  = scale * q_i . k_{g,j}            j over the b block tokens, no mask
 *   m    = max_j s_j,  e_j = exp(s_j - m),  l = sum_j e_j
 *   lin  = phi(q_i) S_g                     (row vector, length d)
 *   default:  y_i = sum_j (e_j / l) v_{g,j} + lin
 *   shared :  y_i = (sum_j e_j v_{g,j} + e^{-m} lin) /
 *                   (l + e^{-m} phi(q_i) . z_g)
 * scale <= 0 selects 1/sqrt(d).  z is read only when shared != 0.  phi is
 * feature map fmap (W: [hkv][d][d], KV head g's projection, for fmap 2).
 */
void oracle_hybrid_step(const double *Q, const double *K, const double *V,
                        const double *S, const double *z, double *Y, long n,
                        long hq, long hkv, long b, long d, double scale,
                        int shared, int fmap, const double *W)
{
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    const long G = hq / hkv;
    long nh;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (nh = 0; nh < n * hq; ++nh) {
        const long ni = nh / hq, h = nh % hq, g = h / G;
        const double *Kg = K + (ni * hkv + g) * b * d;
        const double *Vg = V + (ni * hkv + g) * b * d;
        const double *Sg = S + (ni * hkv + g) * d * d;
        const double *zg = z ? z + (ni * hkv + g) * d : NULL;
        const double *Wg = W ? W + g * d * d : NULL;
        double *s = (double *)malloc(sizeof(double) * (size_t)b);
        double *lin = (double *)malloc(sizeof(double) * (size_t)d);
        double *fq = (double *)malloc(sizeof(double) * (size_t)d);
        for (long i = 0; i < b; ++i) {
            const double *q = Q + ((ni * hq + h) * b + i) * d;
            double *y = Y + ((ni * hq + h) * b + i) * d;
            double m = -INFINITY;
            for (long j = 0; j < b; ++j) {
                double dot = 0.0;
                for (long c = 0; c < d; ++c)
                    dot += q[c] * Kg[j * d + c];
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (long j = 0; j < b; ++j) {
                s[j] = exp(s[j] - m); /* s now holds e_j */
                l += s[j];
            }
            phi_vec(q, d, fmap, Wg, fq);
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long r = 0; r < d; ++r)
                    acc += fq[r] * Sg[r * d + c];
                lin[c] = acc;
            }
            if (!shared) {
                for (long c = 0; c < d; ++c) {
                    double soft = 0.0;
                    for (long j = 0; j < b; ++j)
                        soft += (s[j] / l) * Vg[j * d + c];
                    y[c] = soft + lin[c];
                }
            } else {
                double qz = 0.0;
                for (long r = 0; r < d; ++r)
                    qz += fq[r] * zg[r];
                const double em = exp(-m);
                const double den = l + em * qz;
                for (long c = 0; c < d; ++c) {
                    double num = 0.0;
                    for (long j = 0; j < b; ++j)
                        num += s[j] * Vg[j * d + c];
                    y[c] = (num + em * lin[c]) / den;
                }
            }
        }
        free(s);
        free(lin);
        free(fq);
    }
}

/*
 * Exact prefix softmax (the baseline the abstract describes: every denoising
 * step attends to all previous blocks through the KV cache).  One joint
 * softmax over the P cached tokens followed by the b active-block tokens,
 * bidirectional (no mask):
 *   y_i = sum_j softmax_j(scale * q_i . k_j) v_j,  j in [cache[0:P] || block]
 * Kc, Vc are [n][hkv][cap][d]; K, V are [n][hkv][b][d].
 */
void oracle_prefix_softmax(const double *Q, const double *Kc, const double *Vc,
                           long P, long cap, const double *K, const double *V,
                           double *Y, long n, long hq, long hkv, long b, long d,
                           double scale)
{
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    const long G = hq / hkv;
    const long L = P + b;
    long nh;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (nh = 0; nh < n * hq; ++nh) {
        const long ni = nh / hq, h = nh % hq, g = h / G;
        const double *Kcg = Kc + (ni * hkv + g) * cap * d;
        const double *Vcg = Vc + (ni * hkv + g) * cap * d;
        const double *Kg = K + (ni * hkv + g) * b * d;
        const double *Vg = V + (ni * hkv + g) * b * d;
        double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        for (long i = 0; i < b; ++i) {
            const double *q = Q + ((ni * hq + h) * b + i) * d;
            double *y = Y + ((ni * hq + h) * b + i) * d;
            double m = -INFINITY;
            for (long j = 0; j < L; ++j) {
                const double *k = j < P ? Kcg + j * d : Kg + (j - P) * d;
                double dot = 0.0;
                for (long c = 0; c < d; ++c)
                    dot += q[c] * k[c];
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (long j = 0; j < L; ++j) {
                s[j] = exp(s[j] - m);
                l += s[j];
            }
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long j = 0; j < L; ++j) {
                    const double *v = j < P ? Vcg + j * d : Vg + (j - P) * d;
                    acc += (s[j] / l) * v[c];
                }
                y[c] = acc;
            }
        }
        free(s);
    }
}

/*
 * Reuse of prefix attention for stable tokens, the method of the LoSA page
 * (gist.science explainer of arXiv 2604.12056, section "3. 方法论 LoSA":
 * 局部性剪枝 locality pruning, 缓存复用 cache reuse, 初始化策略 initialisation;
 * and "技术细节" technical details), applied to the exact comparison path with
 * a dense prefix pass over the active tokens (the page's sparse selector,
 * QUEST, is not part of this path).  One denoising step of a block:
 *
 *   1. locality score of block token i of request ni (the MSE of its query
 *      between this denoising step and the previous one, over the token's
 *      whole query: every query head, every dimension):
 *        score_i = (1 / (hq d)) sum_h sum_c (Q[ni][h][i][c] - Qprev[ni][h][i][c])^2
 *   2. the active set A of request ni: the k tokens with the largest score
 *      (ties to the lower token index); the others are stable tokens;
 *   3. for an active token, every query head's prefix attention over the
 *      cache, as a normalised output and its log-normaliser,
 *        o_p = sum_{j<P} e^{s_j} v_j / sum_{j<P} e^{s_j},
 *        lse_p = log sum_{j<P} e^{s_j},       s_j = scale q . k_j,
 *      replaces the token's entries of the cache (O_pre, L_pre); a stable
 *      token keeps the entries of the previous step (the previous step's q);
 *   4. the block's own attention of every token, o_b and lse_b likewise over
 *      the b block tokens with the current q, merged with the cached prefix
 *      part by the online-softmax identity
 *        y = (e^{lse_p - M} o_p + e^{lse_b - M} o_b) / (e^{lse_p - M} + e^{lse_b - M}),
 *        M = max(lse_p, lse_b)      (P = 0: lse_p = -inf, y = o_b).
 * The first denoising step of a block has no cache: every token is active
 * (the page's dense initialisation).  The cache holds b x (d + 1) values per
 * query head, as the page counts.
 */

/* Locality scores and the active set: active[ni * k + a], a < k, lists
 * request ni's active tokens in increasing token order. */
void oracle_losa_select(const double *Q, const double *Qprev, long n, long hq,
                        long b, long d, long k, long *active, double *score)
{
    long ni;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (ni = 0; ni < n; ++ni) {
        double *sc = score + ni * b;
        for (long i = 0; i < b; ++i) {
            /* the squared change summed over groups of 8 columns, the groups
             * of a head, then the heads: each level in index order */
            double acc = 0.0;
            for (long h = 0; h < hq; ++h) {
                const double *q = Q + ((ni * hq + h) * b + i) * d;
                const double *p = Qprev + ((ni * hq + h) * b + i) * d;
                double sh = 0.0;
                for (long c0 = 0; c0 < d; c0 += 8) {
                    double sg = 0.0;
                    for (long c = c0; c < c0 + 8 && c < d; ++c)
                        sg += (q[c] - p[c]) * (q[c] - p[c]);
                    sh += sg;
                }
                acc += sh;
            }
            sc[i] = acc / (double)(hq * d);
        }
        long a = 0;
        for (long i = 0; i < b && a < k; ++i) {
            /* rank of token i: tokens with a larger score, or an equal score
             * and a lower index, come first */
            long rank = 0;
            for (long j = 0; j < b; ++j)
                if (sc[j] > sc[i] || (sc[j] == sc[i] && j < i)) ++rank;
            if (rank < k) active[ni * k + a++] = i;
        }
    }
}

/* Steps 3 and 4 for a given active set (is_active[ni * b + i] != 0): updates
 * O_pre [n][hq][b][d] and L_pre [n][hq][b] for the active tokens, writes Y. */
void oracle_losa_apply(const double *Q, const double *Kc, const double *Vc,
                       long P, long cap, const double *K, const double *V,
                       const long *is_active, double *O_pre, double *L_pre,
                       double *Y, long n, long hq, long hkv, long b, long d,
                       double scale)
{
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    const long G = hq / hkv;
    long nh;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (nh = 0; nh < n * hq; ++nh) {
        const long ni = nh / hq, h = nh % hq, g = h / G;
        const double *Kcg = Kc + (ni * hkv + g) * cap * d;
        const double *Vcg = Vc + (ni * hkv + g) * cap * d;
        const double *Kg = K + (ni * hkv + g) * b * d;
        const double *Vg = V + (ni * hkv + g) * b * d;
        const long L = P > b ? P : b;
        double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        double *ob = (double *)malloc(sizeof(double) * (size_t)d);
        for (long i = 0; i < b; ++i) {
            const long row = (ni * hq + h) * b + i;
            const double *q = Q + row * d;
            double *op = O_pre + row * d;
            if (is_active[ni * b + i]) {
                /* dense prefix pass with this step's q */
                double m = -INFINITY;
                for (long j = 0; j < P; ++j) {
                    double dot = 0.0;
                    for (long c = 0; c < d; ++c)
                        dot += q[c] * Kcg[j * d + c];
                    s[j] = scale * dot;
                    if (s[j] > m) m = s[j];
                }
                double l = 0.0;
                for (long j = 0; j < P; ++j) {
                    s[j] = exp(s[j] - m);
                    l += s[j];
                }
                for (long c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (long j = 0; j < P; ++j)
                        acc += (s[j] / l) * Vcg[j * d + c];
                    op[c] = P > 0 ? acc : 0.0;
                }
                L_pre[row] = P > 0 ? m + log(l) : -INFINITY;
            }
            /* the block's attention with this step's q */
            double mb = -INFINITY;
            for (long j = 0; j < b; ++j) {
                double dot = 0.0;
                for (long c = 0; c < d; ++c)
                    dot += q[c] * Kg[j * d + c];
                s[j] = scale * dot;
                if (s[j] > mb) mb = s[j];
            }
            double lb = 0.0;
            for (long j = 0; j < b; ++j) {
                s[j] = exp(s[j] - mb);
                lb += s[j];
            }
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long j = 0; j < b; ++j)
                    acc += (s[j] / lb) * Vg[j * d + c];
                ob[c] = acc;
            }
            const double lse_b = mb + log(lb);
            const double lse_p = L_pre[row];
            const double M = lse_p > lse_b ? lse_p : lse_b;
            const double wp = lse_p == -INFINITY ? 0.0 : exp(lse_p - M);
            const double wb = exp(lse_b - M);
            double *y = Y + row * d;
            for (long c = 0; c < d; ++c)
                y[c] = (wp * op[c] + wb * ob[c]) / (wp + wb);
        }
        free(ob);
        free(s);
    }
}

/*
 * Block partition of a length-L sequence into blocks of B tokens; the last
 * block may be short (worked example: L=10, B=4 gives tokens 1-4, 5-8, 9-10).
 * Writes the boundaries 0 = bounds[0] < bounds[1] < ... < bounds[k] = L and
 * returns k, the number of blocks (0 for L = 0; -1 for bad arguments).
 * bounds needs room for k + 1 entries.
 */
long oracle_block_partition(long L, long B, long *bounds)
{
    if (L < 0 || B < 1) return -1;
    long k = 0;
    bounds[0] = 0;
    for (long start = 0; start < L; start += B) {
        long end = start + B;
        if (end > L) end = L;
        bounds[++k] = end;
    }
    return k;
}
