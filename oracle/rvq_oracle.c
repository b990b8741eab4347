/*
 * rvq_oracle.c -- plain, slow, fp64 reference for greedy residual vector
 * quantization (RVQ) of visual features, and for its gather-sum decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * bench's CPU-baseline leg load this library.  It shares no code, header,
 * table or helper with the CUDA path.
 *
 * What it computes (LongCat-2.5 technical blog, "Visual Primitive Modeling" ->
 * "Discrete Native Resolution Vision Transformer": RVQ is applied to native-
 * resolution encoder features; Meituan LongCat-2.5 open-source article, section
 * "02 Visual Coding and 3D": the quantizer adds detail level by level; Figure 1
 * of the blog: token sequences are reconstructed by a de-tokenizer; "Offline
 * Visual Preprocessing": the tokenizer is fixed, so ids are a deterministic
 * function of the features):
 *
 *   r = x                                    (fp64, stored values widened exactly)
 *   for l = 0 .. L-1:
 *       d_k  = sum_i (r_i - C_l[k,i])^2      for every k   (direct form)
 *       id_l = smallest k attaining min_k d_k
 *       r    = r - C_l[id_l]
 *   residual = r,   recon = sum_l C_l[id_l]   (ascending l)
 *   decode(ids) = sum_l C_l[ids_l]            (ascending l)
 *
 * Readings where the pages are silent: squared Euclidean distance, greedy
 * choice per level, lowest index on exact ties.
 *
 * Inputs arrive as float32 arrays: every stored value (fp32 or bf16) is exactly
 * representable there, and each element is widened to double before use.
 * Arithmetic is plain double in source order; build with -ffp-contract=off so
 * no multiply-add is fused behind the reader's back.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_ID_RANGE (-5)

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Number of threads a parallel region of this library runs with. */
int rvq_oracle_max_threads(int nthreads)
{
#ifdef _OPENMP
    set_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Squared Euclidean distance between residual r (double) and codeword c. */
static double sq_dist(const double *r, const float *c, int D)
{
    double s = 0.0;
    for (int i = 0; i < D; ++i) {
        double t = r[i] - (double)c[i];
        s += t * t;
    }
    return s;
}

/* Nearest codeword of one level to residual r: returns its index, lowest on ties. */
static int32_t nearest(const double *r, const float *C_l, int K, int D, double *best_d)
{
    int32_t best = 0;
    double bd = sq_dist(r, C_l, D);
    for (int k = 1; k < K; ++k) {
        double d = sq_dist(r, C_l + (size_t)k * D, D);
        if (d < bd) {
            bd = d;
            best = k;
        }
    }
    *best_d = bd;
    return best;
}

/*
 * Greedy RVQ encode of rows x[rows[j]] (or of all N rows when rows == NULL).
 *   x         [N, D]     features
 *   C         [L, K, D]  codebooks
 *   ids       [M, L]     output, M = nrows (or N)
 *   residual  [M, D]     output, may be NULL
 *   recon     [M, D]     output, may be NULL
 *   dist      [M, L]     output, distance of the chosen codeword at each level, may be NULL
 */
int rvq_oracle_encode(const float *x, int64_t N, int D, const float *C, int L, int K,
                      const int64_t *rows, int64_t nrows, int32_t *ids, double *residual,
                      double *recon, double *dist, int nthreads)
{
    if (!x || !C || !ids || D <= 0 || L <= 0 || K <= 0 || N < 0) return ORACLE_ERR_ARG;
    int64_t M = rows ? nrows : N;
    for (int64_t j = 0; rows && j < M; ++j)
        if (rows[j] < 0 || rows[j] >= N) return ORACLE_ERR_ARG;
    set_threads(nthreads);
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *r = (double *)malloc(sizeof(double) * (size_t)D * 2);
        if (!r) {
#pragma omp atomic write
            err = ORACLE_ERR_ARG;
        }
        double *acc = r ? r + D : NULL;
#pragma omp for schedule(dynamic, 1)
        for (int64_t j = 0; j < M; ++j) {
            if (!r) continue;
            int64_t n = rows ? rows[j] : j;
            for (int i = 0; i < D; ++i) {
                r[i] = (double)x[(size_t)n * D + i];
                acc[i] = 0.0;
            }
            for (int l = 0; l < L; ++l) {
                const float *C_l = C + (size_t)l * K * D;
                double bd;
                int32_t id = nearest(r, C_l, K, D, &bd);
                ids[(size_t)j * L + l] = id;
                if (dist) dist[(size_t)j * L + l] = bd;
                const float *c = C_l + (size_t)id * D;
                for (int i = 0; i < D; ++i) {
                    r[i] = r[i] - (double)c[i];
                    acc[i] = acc[i] + (double)c[i];
                }
            }
            if (residual) memcpy(residual + (size_t)j * D, r, sizeof(double) * D);
            if (recon) memcpy(recon + (size_t)j * D, acc, sizeof(double) * D);
        }
        free(r);
    }
    return err;
}

/*
 * Decode: recon[j] = sum_l C_l[ids[j,l]] in ascending l, for M rows of ids.
 * An id outside [0, K) makes the call return ORACLE_ERR_ID_RANGE; that level
 * contributes nothing to its row.
 */
int rvq_oracle_decode(const int32_t *ids, int64_t M, int L, const float *C, int K, int D,
                      double *recon, int nthreads)
{
    if (!ids || !C || !recon || D <= 0 || L <= 0 || K <= 0 || M < 0) return ORACLE_ERR_ARG;
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t j = 0; j < M; ++j) {
        double *out = recon + (size_t)j * D;
        for (int i = 0; i < D; ++i) out[i] = 0.0;
        for (int l = 0; l < L; ++l) {
            int32_t id = ids[(size_t)j * L + l];
            if (id < 0 || id >= K) {
                bad = 1;
                continue;
            }
            const float *c = C + ((size_t)l * K + (size_t)id) * D;
            for (int i = 0; i < D; ++i) out[i] = out[i] + (double)c[i];
        }
    }
    return bad ? ORACLE_ERR_ID_RANGE : ORACLE_OK;
}

/*
 * Validate a given id assignment level by level.  For row x[rows[j]] the residual
 * follows the GIVEN ids (r_0 = x, r_{l+1} = r_l - C_l[ids[j,l]]); at every level the
 * full distance vector to r_l is formed and reported as
 *   best[j,l]    min_k d_k
 *   argmin[j,l]  smallest k attaining it
 *   second[j,l]  min over k != argmin of d_k   (+inf when K == 1)
 *   chosen[j,l]  d at the given id
 * This is the same per-level step as the encode above, driven by ids that some
 * other implementation chose; it lets a caller check that every choice was a
 * nearest codeword even after a legitimate near-tie sent two encoders down
 * different paths.
 */
int rvq_oracle_check_path(const float *x, int64_t N, int D, const float *C, int L, int K,
                          const int64_t *rows, int64_t nrows, const int32_t *ids,
                          double *best, int32_t *argmin, double *second, double *chosen,
                          int nthreads)
{
    if (!x || !C || !ids || !rows || D <= 0 || L <= 0 || K <= 0) return ORACLE_ERR_ARG;
    for (int64_t j = 0; j < nrows; ++j)
        if (rows[j] < 0 || rows[j] >= N) return ORACLE_ERR_ARG;
    for (int64_t j = 0; j < nrows * L; ++j)
        if (ids[j] < 0 || ids[j] >= K) return ORACLE_ERR_ID_RANGE;
    set_threads(nthreads);
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double *r = (double *)malloc(sizeof(double) * (size_t)D);
        double *d = (double *)malloc(sizeof(double) * (size_t)K);
        if (!r || !d) {
#pragma omp atomic write
            err = ORACLE_ERR_ARG;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t j = 0; j < nrows; ++j) {
            if (!r || !d) continue;
            int64_t n = rows[j];
            for (int i = 0; i < D; ++i) r[i] = (double)x[(size_t)n * D + i];
            for (int l = 0; l < L; ++l) {
                const float *C_l = C + (size_t)l * K * D;
                for (int k = 0; k < K; ++k) d[k] = sq_dist(r, C_l + (size_t)k * D, D);
                int32_t a = 0;
                for (int k = 1; k < K; ++k)
                    if (d[k] < d[a]) a = k;
                double s = HUGE_VAL;
                for (int k = 0; k < K; ++k)
                    if (k != a && d[k] < s) s = d[k];
                int32_t g = ids[(size_t)j * L + l];
                size_t o = (size_t)j * L + l;
                best[o] = d[a];
                argmin[o] = a;
                second[o] = s;
                chosen[o] = d[g];
                const float *c = C_l + (size_t)g * D;
                for (int i = 0; i < D; ++i) r[i] = r[i] - (double)c[i];
            }
        }
        free(r);
        free(d);
    }
    return err;
}

/* d[k] = sum_i (r_i - C_l[k,i])^2 for k in [0, K): the distance vector of one level. */
int rvq_oracle_distances(const double *r, const float *C_l, int K, int D, double *d)
{
    if (!r || !C_l || !d || K <= 0 || D <= 0) return ORACLE_ERR_ARG;
    for (int k = 0; k < K; ++k) d[k] = sq_dist(r, C_l + (size_t)k * D, D);
    return ORACLE_OK;
}

/*
 * Gradient of the visual-token embedding of the backbone (LongCat-2.5 technical blog,
 * "Visual Primitive Modeling": the visual codebook embeddings are learned jointly with the
 * backbone).  The embedding of a token is the same gather-sum as decode, with learned tables E:
 *     e[n] = sum_l E_l[ids[n,l]]
 * so its gradient with respect to the tables, given g = dLoss/de [N,H], is
 *     grad[l, k, :] = sum over n with ids[n,l] == k of g[n, :]
 * accumulated here in fp64, in ascending n, into the caller's array (zero it for a fresh
 * gradient).  count[l,k] (optional) receives the number of such n, absum[l,k,:] (optional) the
 * sum of |g[n,:]| over them: the magnitudes that bound the rounding of an fp32 sum of the same
 * terms taken in any order.  An id outside [0, K) returns ORACLE_ERR_ID_RANGE and adds nothing.
 * Parallel over levels only, so every (l, k) row is summed by one thread in row order.
 */
int rvq_oracle_embed_backward(const int32_t *ids, int64_t N, int L, int K, int H, const float *g,
                              double *grad, int64_t *count, double *absum, int nthreads)
{
    if (!ids || !g || !grad || H <= 0 || L <= 0 || K <= 0 || N < 0) return ORACLE_ERR_ARG;
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int l = 0; l < L; ++l) {
        for (int64_t n = 0; n < N; ++n) {
            int32_t id = ids[(size_t)n * L + l];
            if (id < 0 || id >= K) {
                bad = 1;
                continue;
            }
            double *dst = grad + ((size_t)l * K + (size_t)id) * H;
            const float *src = g + (size_t)n * H;
            for (int i = 0; i < H; ++i) dst[i] = dst[i] + (double)src[i];
            if (count) count[(size_t)l * K + (size_t)id] += 1;
            if (absum) {
                double *a = absum + ((size_t)l * K + (size_t)id) * H;
                for (int i = 0; i < H; ++i) a[i] = a[i] + fabs((double)src[i]);
            }
        }
    }
    return bad ? ORACLE_ERR_ID_RANGE : ORACLE_OK;
}

/*
 * One Lloyd (k-means) update of one codebook level, the step that fits the fixed tokenizer the
 * blog's "Offline Visual Preprocessing" relies on (the pages do not describe fitting; reading:
 * plain k-means on the level's input residuals, an empty cluster keeps its codeword).  Given the
 * level's input points p [N,D] (the residuals r_l the encode saw at this level) and their
 * assignments ids [N] (the level's chosen codewords):
 *     count[k]  = #{n : ids[n] == k}
 *     new[k, :] = (1 / count[k]) * sum over those n of p[n, :]      (fp64, ascending n)
 *     new[k, :] = old[k, :]                                           when count[k] == 0
 * absum[k,:] (optional) = sum of |p[n,:]| over the cluster, for a rounding bound on an fp32 sum.
 * An id outside [0, K) returns ORACLE_ERR_ID_RANGE and the row is ignored.
 */
int rvq_oracle_codebook_update(const float *p, const int32_t *ids, int64_t N, int D, int K, const float *old_cb,
                               double *new_cb, int64_t *count, double *absum)
{
    if (!p || !ids || !old_cb || !new_cb || !count || D <= 0 || K <= 0 || N < 0) return ORACLE_ERR_ARG;
    int bad = 0;
    for (size_t i = 0; i < (size_t)K * D; ++i) new_cb[i] = 0.0;
    if (absum)
        for (size_t i = 0; i < (size_t)K * D; ++i) absum[i] = 0.0;
    for (int k = 0; k < K; ++k) count[k] = 0;
    for (int64_t n = 0; n < N; ++n) {
        int32_t id = ids[n];
        if (id < 0 || id >= K) {
            bad = 1;
            continue;
        }
        double *s = new_cb + (size_t)id * D;
        const float *x = p + (size_t)n * D;
        for (int i = 0; i < D; ++i) s[i] = s[i] + (double)x[i];
        if (absum) {
            double *a = absum + (size_t)id * D;
            for (int i = 0; i < D; ++i) a[i] = a[i] + fabs((double)x[i]);
        }
        count[id] += 1;
    }
    for (int k = 0; k < K; ++k) {
        double *s = new_cb + (size_t)k * D;
        if (count[k] == 0) {
            for (int i = 0; i < D; ++i) s[i] = (double)old_cb[(size_t)k * D + i];
        } else {
            for (int i = 0; i < D; ++i) s[i] = s[i] / (double)count[k];
        }
    }
    return bad ? ORACLE_ERR_ID_RANGE : ORACLE_OK;
}

/*
 * Balance pretokenized image sequences across data-parallel ranks by visual-token count
 * (LongCat-2.5 technical blog, "Offline Visual Preprocessing" and "Supernode-Aware Parallelism":
 * with ids precomputed, every image's token count is known when batches are packed, which keeps
 * the load even across data-parallel ranks; the pages give no algorithm, the reading is the
 * classic longest-processing-time-first rule).  Sequences are taken in decreasing length (equal
 * lengths: lower index first) and each goes to the rank with the smallest load so far (equal
 * loads: lower rank).  owner[s] receives the rank of sequence s, load[r] the tokens of rank r.
 * Plain O(S log S + S * world) loops.
 */
int rvq_oracle_balance(const int64_t *lengths, int64_t S, int world, int32_t *owner, int64_t *load)
{
    if (!lengths || !owner || !load || S < 0 || world < 1) return ORACLE_ERR_ARG;
    for (int64_t s = 0; s < S; ++s)
        if (lengths[s] < 0) return ORACLE_ERR_ARG;
    int64_t *order = (int64_t *)malloc((size_t)(S > 0 ? S : 1) * sizeof(int64_t));
    if (!order) return ORACLE_ERR_ARG;
    for (int64_t s = 0; s < S; ++s) order[s] = s;
    /* insertion sort: decreasing length, then increasing index (stable on the index order) */
    for (int64_t i = 1; i < S; ++i) {
        int64_t v = order[i], j = i - 1;
        while (j >= 0 && lengths[order[j]] < lengths[v]) {
            order[j + 1] = order[j];
            --j;
        }
        order[j + 1] = v;
    }
    for (int r = 0; r < world; ++r) load[r] = 0;
    for (int64_t i = 0; i < S; ++i) {
        int best = 0;
        for (int r = 1; r < world; ++r)
            if (load[r] < load[best]) best = r;
        owner[order[i]] = best;
        load[best] += lengths[order[i]];
    }
    free(order);
    return ORACLE_OK;
}
