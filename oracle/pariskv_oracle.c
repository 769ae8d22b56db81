/*
 * pariskv_oracle.c -- plain, slow CPU oracle for the ParisKV KV-cache retrieval path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load or call this file. It shares no code, header, table or helper
 * with the CUDA library: every step below is written out from its definition, in the order
 * the method states it, without blocking, fusion or reordering.
 *
 * Sources (cited by page title and section):
 *   [TS]  "Technical Summary: ParisKV" (gist.science/paper/2602.07721)
 *   [ABS] "ParisKV: Fast and Drift-Robust KV-Cache Retrieval for Long-Context LLMs"
 *         (ICML 2026 poster page, abstract)
 *
 * Precision. The rotation and the attention reference run in fp64 (the pages fix no
 * precision for them). The steps that decide integers or rankings from the rotated fp32
 * vectors (bucket ids, 4-bit codes, calibration factors, query lookup table, vote scores,
 * rerank estimates, selections) are fixed-order fp32 computations, because the GPU path must
 * reproduce them bit for bit from identical rotated fp32 inputs. Build with
 * -ffp-contract=off and without fast-math so that every a*b+c below is two roundings unless
 * it is written as fmaf().
 *
 * Readings of points the pages leave open are marked [R#]; each one is listed with its
 * justification in the design notes of this repository.
 *
 * Layouts (canonical, row-major): keys/queries [n][d] f32; ids [n][B] u8; code magnitudes
 * [n][d] i32; code sign bits [n][d] u8; factors [n][B] f32; lookup table [B][2^m] u8.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of OpenMP threads the oracle will use (1 without OpenMP). */
int32_t orc_num_threads(void)
{
#ifdef _OPENMP
    return (int32_t)omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int32_t t)
{
#ifdef _OPENMP
    if (t > 0) omp_set_num_threads(t);
#else
    (void)t;
#endif
}

/* ------------------------------------------------------------------------------------
 * Rotation. [TS] Methodology, Core Algorithmic Innovations 1, "Normalization and
 * Rotation": keys and queries are l2-normalised, then rotated by one shared random
 * orthogonal rotation implemented as an SRHT.
 *
 * [R1] R = (1/sqrt(d)) * H * diag(s): H is the Sylvester-ordered Walsh-Hadamard matrix,
 *      H[i][j] = (-1)^popcount(i & j); s[j] in {+1,-1} is the random sign vector (an input).
 *      No subsampling: the rotated vector keeps all d coordinates.
 * ------------------------------------------------------------------------------------ */
static int hadamard_entry(int64_t i, int64_t j)
{
    return (__builtin_popcountll((unsigned long long)(i & j)) & 1) ? -1 : 1;
}

/* y = R x in fp64, written as the explicit d x d matrix-vector product. */
void orc_rotate_f64(int32_t d, const int8_t* signs, const double* x, double* y)
{
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int32_t i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int32_t j = 0; j < d; ++j)
            acc += (double)hadamard_entry(i, j) * (double)signs[j] * x[j];
        y[i] = acc * inv_sqrt_d;
    }
}

/* [R3] Normalise then rotate, per row: norm = ||x||_2 (fp64), xhat = x / norm,
 * y = R xhat rounded to fp32, norm rounded to fp32. A zero row gives y = 0, norm = 0. */
void orc_normalize_rotate(int32_t d, const int8_t* signs, const float* x, int64_t n,
                          float* y, float* norm)
{
#pragma omp parallel
    {
        double* xh = (double*)malloc(sizeof(double) * (size_t)d);
        double* yr = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < n; ++r) {
            const float* xr = x + r * d;
            double ss = 0.0;
            for (int32_t j = 0; j < d; ++j) ss += (double)xr[j] * (double)xr[j];
            double nr = sqrt(ss);
            if (nr == 0.0) {
                for (int32_t j = 0; j < d; ++j) y[r * d + j] = 0.0f;
                norm[r] = 0.0f;
                continue;
            }
            for (int32_t j = 0; j < d; ++j) xh[j] = (double)xr[j] / nr;
            orc_rotate_f64(d, signs, xh, yr);
            for (int32_t j = 0; j < d; ++j) y[r * d + j] = (float)yr[j];
            norm[r] = (float)nr;
        }
        free(xh);
        free(yr);
    }
}

/* ------------------------------------------------------------------------------------
 * Key encoding from rotated fp32 vectors.
 *
 * Bucket ids. [TS] Core Algorithmic Innovations 1 "Analytic Centroids" and 2 "Coarse
 * Candidate Generation": the rotated key is split into B subspaces of m dims; each subspace
 * direction is assigned to its nearest analytic sign centroid (coordinates +-1/sqrt(m)).
 * All centroids have the same norm, so the nearest one is the one with the largest inner
 * product, i.e. the sign pattern of the subspace.
 * [R4] bit j of id_b is (y[b*m+j] < 0): the first dim is the least significant bit, and a
 *      zero (or -0) coordinate gives bit 0, which is the lower id of the tie.
 *
 * RSQ codes. [TS] Candidate Reranking (RSQ-IP), "Quantization": a 4-bit code per dim, one
 * sign bit and three magnitude bits.
 * [R5] Magnitudes are uniform levels over [0, mx_b], mx_b = max_j |y_{b,j}|:
 *      mag_j = mx_b == 0 ? 0 : min(L, floorf((L * |y_j|) / mx_b + 0.5f)), L = 7 for 3 bits
 *      (the convergence check uses larger L). Sign bit = (y_j < 0). The dequantised integer
 *      vector is vt_j = (sign ? -1 : +1) * mag_j.
 *
 * Calibration factor. [TS] Candidate Reranking, "Calibration" and "Estimation": a
 * per-(key, subspace) scale w_{i,b} corrects the alignment error of the quantised
 * direction, and <k,q> ~ ||q|| sum_b w_{i,b} <v_{i,b}, q~_b>.
 * [R6] w_{i,b} = ||k_i|| * ||y_b|| / <u_b, v_b> with u_b = y_b/||y_b||, v_b = vt_b/||vt_b||.
 *      Folding the normalisations of v_b into the stored factor gives
 *      f_{i,b} = (||k|| * n2_b) / dot_b,  n2_b = sum_j y_j^2,  dot_b = sum_j vt_j * y_j,
 *      so that f_{i,b} * <vt_b, q~_b> = w_{i,b} * <v_b, q~_b>. Both sums are fmaf chains over
 *      j ascending from 0.0f; f = 0 when dot_b == 0 (an all-zero subspace).
 * ------------------------------------------------------------------------------------ */
void orc_encode_rotated(int32_t d, int32_t m, int32_t levels, const float* y, const float* knorm,
                        int64_t n, uint8_t* ids, int32_t* mag, uint8_t* neg, float* factor)
{
    const int32_t B = d / m;
    const float Lf = (float)levels;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int32_t b = 0; b < B; ++b) {
            const float* yb = y + r * d + (int64_t)b * m;
            uint32_t id = 0;
            float mx = 0.0f;
            for (int32_t j = 0; j < m; ++j) {
                if (yb[j] < 0.0f) id |= 1u << j;
                float a = fabsf(yb[j]);
                if (a > mx) mx = a;
            }
            ids[r * B + b] = (uint8_t)id;

            float n2 = 0.0f, dot = 0.0f;
            for (int32_t j = 0; j < m; ++j) {
                const int64_t o = r * d + (int64_t)b * m + j;
                int32_t q = 0;
                if (mx != 0.0f) {
                    float t = Lf * fabsf(yb[j]);
                    t = t / mx;
                    t = t + 0.5f;
                    q = (int32_t)floorf(t);
                    if (q > levels) q = levels;
                }
                mag[o] = q;
                neg[o] = (uint8_t)(yb[j] < 0.0f);
                float vt = neg[o] ? -(float)q : (float)q;
                n2 = fmaf(yb[j], yb[j], n2);
                dot = fmaf(vt, yb[j], dot);
            }
            float num = knorm[r] * n2;
            factor[r * B + b] = (dot == 0.0f) ? 0.0f : num / dot;
        }
    }
}

/* ------------------------------------------------------------------------------------
 * RSQ codes with a level table ("Beta-prior" levels). [TS] Core Algorithmic Innovations 2,
 * "Quantization": the 3-bit magnitudes are "derived from rotation-induced Beta priors".
 * [R24] Levels c_0 < ... < c_7 (fp32, a table given as input) for the ratio
 *       r_j = |y_j| / max_i |y_i| of the subspace; thresholds t_i = fp32 of the exact
 *       midpoint (c_{i-1} + c_i) / 2; mag_j = number of i in 1..7 with r_j >= t_i (r_j in
 *       IEEE fp32: |y_j| / max); the signed level vt_j = (y_j < 0 ? -c : c)[mag_j]. The
 *       factor is the same fold as with uniform levels, f = ||k|| * sum y^2 / sum vt y (fp32
 *       FMA chains, j ascending), 0 for an all-zero subspace.
 * ------------------------------------------------------------------------------------ */
void orc_encode_rotated_table(int32_t d, int32_t m, const float* lv, const float* y,
                              const float* knorm, int64_t n, uint8_t* ids, int32_t* mag,
                              uint8_t* neg, float* factor)
{
    const int32_t B = d / m;
    float th[8];
    for (int32_t i = 1; i < 8; ++i) th[i] = (float)(((double)lv[i - 1] + (double)lv[i]) * 0.5);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int32_t b = 0; b < B; ++b) {
            const float* yb = y + r * d + (int64_t)b * m;
            uint32_t id = 0;
            float mx = 0.0f;
            for (int32_t j = 0; j < m; ++j) {
                if (yb[j] < 0.0f) id |= 1u << j;
                float a = fabsf(yb[j]);
                if (a > mx) mx = a;
            }
            ids[r * B + b] = (uint8_t)id;
            float n2 = 0.0f, dot = 0.0f;
            for (int32_t j = 0; j < m; ++j) {
                const int64_t o = r * d + (int64_t)b * m + j;
                int32_t q = 0;
                if (mx != 0.0f) {
                    const float ratio = fabsf(yb[j]) / mx;
                    for (int32_t i = 1; i < 8; ++i) q += ratio >= th[i];
                }
                mag[o] = q;
                neg[o] = (uint8_t)(yb[j] < 0.0f);
                const float vt = neg[o] ? -lv[q] : lv[q];
                n2 = fmaf(yb[j], yb[j], n2);
                dot = fmaf(vt, yb[j], dot);
            }
            const float num = knorm[r] * n2;
            factor[r * B + b] = (dot == 0.0f) ? 0.0f : num / dot;
        }
    }
}

/* The rerank of orc_rerank with table levels: vt_j = (neg ? -lv : lv)[mag_j], same chains. */
void orc_rerank_table(int32_t d, int32_t m, const float* lv, const int32_t* mag,
                      const uint8_t* neg, const float* factor, const int32_t* cand, int64_t C,
                      const float* qt, float* S)
{
    const int32_t B = d / m;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        const int64_t i = cand[c];
        float s = 0.0f;
        for (int32_t b = 0; b < B; ++b) {
            float p = 0.0f;
            for (int32_t j = 0; j < m; ++j) {
                const int64_t o = i * d + (int64_t)b * m + j;
                const float vt = neg[o] ? -lv[mag[o]] : lv[mag[o]];
                p = fmaf(vt, qt[(int64_t)b * m + j], p);
            }
            s = fmaf(factor[i * B + b], p, s);
        }
        S[c] = s;
    }
}

/* ------------------------------------------------------------------------------------
 * Query lookup table. [TS] "Coarse Candidate Generation": for a query, each subspace
 * selects the top-rho centroids most similar to the rotated query subspace; keys in those
 * buckets get tiered votes.
 * Similarity: <q~_b, c> * sqrt(m) = sum_j |q~_j| - 2 * penalty(c), where penalty(c) is the
 * sum of |q~_j| over the bits j in which c differs from the query's own sign pattern c1.
 * [R7] penalty is an fp32 sum over j ascending, from 0.0f; centroids are ranked by
 *      (penalty ascending, id ascending) and the first rho are selected.
 * [R8] Tiered weights: rank 1 gets w_rank1 (2), ranks 2..rho get w_rest (1), others 0.
 * ------------------------------------------------------------------------------------ */
typedef struct {
    float pen;
    int32_t id;
} pen_entry;

static int cmp_pen(const void* a, const void* b)
{
    const pen_entry* x = (const pen_entry*)a;
    const pen_entry* y = (const pen_entry*)b;
    if (x->pen < y->pen) return -1;
    if (x->pen > y->pen) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

void orc_query_lut(int32_t d, int32_t m, int32_t rho, int32_t w_rank1, int32_t w_rest,
                   const float* qt, uint8_t* lut)
{
    const int32_t B = d / m;
    const int32_t nc = 1 << m;
    pen_entry* e = (pen_entry*)malloc(sizeof(pen_entry) * (size_t)nc);
    for (int32_t b = 0; b < B; ++b) {
        const float* qb = qt + (int64_t)b * m;
        uint32_t c1 = 0;
        for (int32_t j = 0; j < m; ++j)
            if (qb[j] < 0.0f) c1 |= 1u << j;
        for (int32_t c = 0; c < nc; ++c) {
            float pen = 0.0f;
            uint32_t diff = (uint32_t)c ^ c1;
            for (int32_t j = 0; j < m; ++j)
                if ((diff >> j) & 1u) pen = pen + fabsf(qb[j]);
            e[c].pen = pen;
            e[c].id = c;
        }
        qsort(e, (size_t)nc, sizeof(pen_entry), cmp_pen);
        uint8_t* lb = lut + (int64_t)b * nc;
        for (int32_t c = 0; c < nc; ++c) lb[c] = 0;
        for (int32_t r = 0; r < rho && r < nc; ++r)
            lb[e[r].id] = (uint8_t)(r == 0 ? w_rank1 : w_rest);
    }
    free(e);
}

/* ------------------------------------------------------------------------------------
 * Learned centroids (the comparator of the drift claim). [TS] Problem Statement 2
 * ("Decoding Drift": centroids learned by clustering prefill keys go stale as decoding keys
 * accumulate) and Key Contributions 1 (analytic centroids remove the need for them).
 * [R25] The comparator replaces only the coarse stage's centroids: per (unit, subspace) 256
 *       centroids mu_c in R^8 learned from the prefill keys' rotated subspace vectors.
 *       A key's id is argmax_c <y_b, mu_c> (fp32 FMA chain over j ascending from 0.0f;
 *       ties to the lower c); a query's top-rho are the rho largest <q~_b, mu_c> (same
 *       chain; ties to the lower c), with the tiered weights of [R8]. Everything else (codes,
 *       factors, vote, candidates, rerank, top-k) is unchanged.
 * cent: [B][256][m] for one unit.
 * ------------------------------------------------------------------------------------ */
static float dot_chain(const float* a, const float* b, int32_t m)
{
    float s = 0.0f;
    for (int32_t j = 0; j < m; ++j) s = fmaf(a[j], b[j], s);
    return s;
}

void orc_learned_ids(int32_t d, int32_t m, const float* cent, const float* y, int64_t n,
                     uint8_t* ids)
{
    const int32_t B = d / m, nc = 1 << m;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int32_t b = 0; b < B; ++b) {
            const float* yb = y + r * d + (int64_t)b * m;
            const float* cb = cent + (int64_t)b * nc * m;
            float best = dot_chain(cb, yb, m);
            int32_t arg = 0;
            for (int32_t c = 1; c < nc; ++c) {
                const float v = dot_chain(cb + (int64_t)c * m, yb, m);
                if (v > best) { best = v; arg = c; }
            }
            ids[r * B + b] = (uint8_t)arg;
        }
    }
}

typedef struct {
    float s;
    int32_t id;
} sim_entry;

static int cmp_sim(const void* a, const void* b)
{
    const sim_entry* x = (const sim_entry*)a;
    const sim_entry* y = (const sim_entry*)b;
    if (x->s != y->s) return (x->s < y->s) ? 1 : -1;
    return (x->id > y->id) - (x->id < y->id);
}

void orc_learned_lut(int32_t d, int32_t m, int32_t rho, int32_t w_rank1, int32_t w_rest,
                     const float* cent, const float* qt, uint8_t* lut)
{
    const int32_t B = d / m, nc = 1 << m;
    sim_entry* e = (sim_entry*)malloc(sizeof(sim_entry) * (size_t)nc);
    for (int32_t b = 0; b < B; ++b) {
        const float* cb = cent + (int64_t)b * nc * m;
        for (int32_t c = 0; c < nc; ++c) {
            e[c].s = dot_chain(cb + (int64_t)c * m, qt + (int64_t)b * m, m);
            e[c].id = c;
        }
        qsort(e, (size_t)nc, sizeof(sim_entry), cmp_sim);
        uint8_t* lb = lut + (int64_t)b * nc;
        for (int32_t c = 0; c < nc; ++c) lb[c] = 0;
        for (int32_t r = 0; r < rho && r < nc; ++r)
            lb[e[r].id] = (uint8_t)(r == 0 ? w_rank1 : w_rest);
    }
    free(e);
}

/* Collision vote. [TS] "Coarse Candidate Generation": votes are summed over subspaces into
 * an integer coarse score: score_i = sum_b lut[b][id_{i,b}]. */
void orc_vote(int32_t B, int32_t m, const uint8_t* ids, int64_t n, const uint8_t* lut,
              int32_t* score)
{
    const int32_t nc = 1 << m;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int32_t s = 0;
        for (int32_t b = 0; b < B; ++b) s += lut[(int64_t)b * nc + ids[i * B + b]];
        score[i] = s;
    }
}

/* ------------------------------------------------------------------------------------
 * Candidate pruning. [TS] "Coarse Candidate Generation": the coarse score prunes the
 * search to a small candidate set, e.g. the top 5-10%.
 * [R10] C = min(n, max(k, ceil(n * bp / 10000))), bp the fraction in basis points.
 * The candidates are the first C keys when all keys are ordered by (score descending,
 * index ascending); they are returned in ascending index order.
 * ------------------------------------------------------------------------------------ */
int64_t orc_candidate_count(int64_t n, int64_t k, int32_t bp)
{
    int64_t c = (n * (int64_t)bp + 9999) / 10000;
    if (c < k) c = k;
    if (c > n) c = n;
    return c;
}

typedef struct {
    int32_t score;
    int32_t idx;
} score_entry;

static int cmp_score_desc(const void* a, const void* b)
{
    const score_entry* x = (const score_entry*)a;
    const score_entry* y = (const score_entry*)b;
    if (x->score != y->score) return (x->score < y->score) ? 1 : -1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int cmp_i32(const void* a, const void* b)
{
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

void orc_select_candidates(const int32_t* score, int64_t n, int64_t C, int32_t* cand)
{
    score_entry* e = (score_entry*)malloc(sizeof(score_entry) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        e[i].score = score[i];
        e[i].idx = (int32_t)i;
    }
    qsort(e, (size_t)n, sizeof(score_entry), cmp_score_desc);
    for (int64_t i = 0; i < C; ++i) cand[i] = e[i].idx;
    qsort(cand, (size_t)C, sizeof(int32_t), cmp_i32);
    free(e);
}

/* ------------------------------------------------------------------------------------
 * RSQ-IP rerank. [TS] Candidate Reranking, "Estimation": <k,q> is estimated as
 * ||q|| * sum_b w_{i,b} <v_{i,b}, q~_b> from the codes and factors alone.
 * [R11] p_b = fmaf chain over j ascending of vt_j * q~_{b,j} from 0.0f;
 *       S = fmaf chain over b ascending of f_b * p_b from 0.0f. The ranking uses S
 *       (the estimate divided by ||q||); est = ||q|| * S.
 * ------------------------------------------------------------------------------------ */
void orc_rerank(int32_t d, int32_t m, const int32_t* mag, const uint8_t* neg,
                const float* factor, const int32_t* cand, int64_t C, const float* qt, float* S)
{
    const int32_t B = d / m;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        const int64_t i = cand[c];
        float s = 0.0f;
        for (int32_t b = 0; b < B; ++b) {
            float p = 0.0f;
            for (int32_t j = 0; j < m; ++j) {
                const int64_t o = i * d + (int64_t)b * m + j;
                float vt = neg[o] ? -(float)mag[o] : (float)mag[o];
                p = fmaf(vt, qt[(int64_t)b * m + j], p);
            }
            s = fmaf(factor[i * B + b], p, s);
        }
        S[c] = s;
    }
}

/* ------------------------------------------------------------------------------------
 * Final top-k. [TS] Problem Statement (attention over a Top-k subset) and Key Contributions
 * 2 (Top-k selection on compressed codes); [ABS] (on-demand top-k fetching).
 * [R12] The k candidates with the largest S, ties to the lower key index; returned in
 *       ascending index order together with their S.
 * ------------------------------------------------------------------------------------ */
typedef struct {
    float s;
    int32_t idx;
} est_entry;

static int cmp_est_desc(const void* a, const void* b)
{
    const est_entry* x = (const est_entry*)a;
    const est_entry* y = (const est_entry*)b;
    if (x->s != y->s) return (x->s < y->s) ? 1 : -1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int cmp_est_idx(const void* a, const void* b)
{
    const est_entry* x = (const est_entry*)a;
    const est_entry* y = (const est_entry*)b;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

void orc_topk(const float* S, const int32_t* cand, int64_t C, int64_t k, int32_t* idx_out,
              float* s_out)
{
    est_entry* e = (est_entry*)malloc(sizeof(est_entry) * (size_t)(C > 0 ? C : 1));
    for (int64_t i = 0; i < C; ++i) {
        e[i].s = S[i];
        e[i].idx = cand[i];
    }
    qsort(e, (size_t)C, sizeof(est_entry), cmp_est_desc);
    if (k > C) k = C;
    qsort(e, (size_t)k, sizeof(est_entry), cmp_est_idx);
    for (int64_t i = 0; i < k; ++i) {
        idx_out[i] = e[i].idx;
        s_out[i] = e[i].s;
    }
    free(e);
}

/* ------------------------------------------------------------------------------------
 * Sparse decode attention. [TS] Problem Statement (attend only to a Top-k subset of past
 * tokens) and System-Level Innovations 1 (the selected full-precision K/V rows are fetched).
 * [R13] o = sum_{t in topk} softmax_t(scale * <q, K_t>) V_t over exactly the top-k rows,
 *       in fp64. K and V rows are given as fp32 (exact widening of bf16 inputs).
 * ------------------------------------------------------------------------------------ */
void orc_attend(int32_t d, const float* q, const float* K, const float* V, const int32_t* idx,
                int64_t k, double scale, double* out)
{
    double* l = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    double mx = -INFINITY;
    for (int64_t t = 0; t < k; ++t) {
        const float* kr = K + (int64_t)idx[t] * d;
        double acc = 0.0;
        for (int32_t j = 0; j < d; ++j) acc += (double)q[j] * (double)kr[j];
        l[t] = scale * acc;
        if (l[t] > mx) mx = l[t];
    }
    double den = 0.0;
    for (int32_t j = 0; j < d; ++j) out[j] = 0.0;
    for (int64_t t = 0; t < k; ++t) {
        double w = exp(l[t] - mx);
        den += w;
        const float* vr = V + (int64_t)idx[t] * d;
        for (int32_t j = 0; j < d; ++j) out[j] += w * (double)vr[j];
    }
    for (int32_t j = 0; j < d; ++j) out[j] = (k > 0) ? out[j] / den : 0.0;
    free(l);
}
