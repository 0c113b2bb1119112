/*
 * Reference oracle for InstaGen group-shared importance-sampled permuted
 * block-sparse attention (one DiT self-attention call, per head).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, obviously correct CPU
 * statement of what the GPU path computes.  Only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may load it; the product path never does.
 * It shares no code, header, table or constant generator with the CUDA library.
 *
 * Sources (web pages on "InstaGen: Group-Shared Importance Sampling for Fast
 * Video Generation", arXiv 2611.08610):
 *   [ABS]   the paper's abstract (paper-reading aggregator page and the
 *           thelatestinai.com paper page): block selection treated as an
 *           importance-sampling problem; the highest-scoring keys are attended
 *           exactly; the others enter through a sample whose draw probability
 *           follows their estimated attention, each sampled score weighted by
 *           the inverse of that probability; one sample per query cluster,
 *           used by every query in it.
 *   [FIG3]  thelatestinai.com paper page, Figure 3 caption: (a) clustering
 *           of both queries and keys; (b) from centroid scores, a probability
 *           pi per key group for each query group; (c) the first-ranked key
 *           group is never dropped, the other keys are drawn with probability
 *           following pi and weighted by 1/pi; (d) one key list per query
 *           group, so a single kernel works on dense tiles.
 *   [FIG2]  same page, Figure 2 caption: SVG2 clustering configuration
 *           Cq = 100 query and Ck = 500 key clusters.
 *   [ICLR]  acceptodds.com ICLR 2027 listing, abstract: every query of the
 *           cluster uses the same sample; sampled keys and top-k blocks go
 *           through one attention kernel, and the weights on the sampled
 *           scores make them represent all of the skipped keys.
 *
 * Where the pages are silent the plainest reading is taken; each such reading
 * is marked "[reading]" below.
 *
 * Floating point: everything that decides an integer (scores, ranking, the
 * integer sampling weights) uses single-precision operations that are
 * correctly rounded (multiply, add, fmaf, floorf, ldexpf), so any conforming
 * implementation reaches the same bits.  Build with -ffp-contract=off.
 * Everything else (distances, means, softmax, log-weights) is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NOMEM 2

/* ------------------------------------------------------------------------- */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy
 * as 1, 2, 3", SC 2011).  Round: two 32x32->64 multiplies by the Philox
 * multipliers, outputs permuted and xored with the key; the key is bumped by
 * the Weyl constants (golden ratio and sqrt(3)-1 in 32-bit fixed point)
 * between rounds.  Ten rounds.                                               */
/* ------------------------------------------------------------------------- */
void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    const uint32_t mul0 = 0xD2511F53u, mul1 = 0xCD9E8D57u;
    const uint32_t weyl0 = 0x9E3779B9u, weyl1 = 0xBB67AE85u;
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += weyl0; k1 += weyl1; }
        uint64_t p0 = (uint64_t)mul0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)mul1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Batch form used by the tests: ctrs [n,4], keys [n,2] -> out [n,4]. */
void orc_philox_batch(int64_t n, const uint32_t* ctrs, const uint32_t* keys, uint32_t* out)
{
    for (int64_t i = 0; i < n; ++i) orc_philox4x32_10(ctrs + 4 * i, keys + 2 * i, out + 4 * i);
}

/* ------------------------------------------------------------------------- */
/* Budgets.  [reading] E and m are the given shares of the N keys rounded to
 * the nearest integer, halves away from zero (Table 1 caption of the paper
 * page: E + S names the exactly attended plus the sampled key fraction of a
 * sparse call).                                                              */
/* ------------------------------------------------------------------------- */
int64_t orc_budget(float frac, int64_t N)
{
    return (int64_t)llround((double)frac * (double)N);
}

/* ------------------------------------------------------------------------- */
/* (a) k-means clustering of one head's queries or keys [FIG3 (a)].
 * [reading] squared Euclidean distance; initial centroid j is token
 * floor(j*N/C); ties go to the lowest centroid index; an empty cluster keeps
 * its previous centroid; T Lloyd iterations of (assign, update), so the
 * returned centroids are the means of the returned clusters.                */
/* ------------------------------------------------------------------------- */
void orc_kmeans_init(const float* X, int64_t N, int d, int C, float* cent)
{
    for (int j = 0; j < C; ++j) {
        int64_t src = ((int64_t)j * N) / C;
        memcpy(cent + (int64_t)j * d, X + src * d, sizeof(float) * (size_t)d);
    }
}

/* assign[i] = argmin_j ||x_i - c_j||^2 in fp64, lowest j on ties.
 * inertia (optional) = sum_i min_j ||x_i - c_j||^2.                          */
void orc_kmeans_assign(const float* X, int64_t N, int d, const float* cent, int C,
                       int32_t* assign, double* inertia)
{
    double total = 0.0;
    #pragma omp parallel for schedule(static) reduction(+:total)
    for (int64_t i = 0; i < N; ++i) {
        const float* x = X + i * d;
        double best = INFINITY;
        int32_t best_j = 0;
        for (int j = 0; j < C; ++j) {
            const float* c = cent + (int64_t)j * d;
            double dist = 0.0;
            for (int k = 0; k < d; ++k) {
                double diff = (double)x[k] - (double)c[k];
                dist += diff * diff;
            }
            if (dist < best) { best = dist; best_j = j; }
        }
        assign[i] = best_j;
        total += best;
    }
    if (inertia) *inertia = total;
}

/* c_j = mean of its members (fp64 sum in ascending token order, rounded to
 * fp32); an empty cluster keeps its centroid.                               */
int orc_kmeans_update(const float* X, int64_t N, int d, const int32_t* assign, int C, float* cent)
{
    double* sums = (double*)calloc((size_t)C * (size_t)d, sizeof(double));
    int64_t* counts = (int64_t*)calloc((size_t)C, sizeof(int64_t));
    if (!sums || !counts) { free(sums); free(counts); return ORC_ERR_NOMEM; }
    for (int64_t i = 0; i < N; ++i) {
        int32_t a = assign[i];
        if (a < 0 || a >= C) { free(sums); free(counts); return ORC_ERR_ARG; }
        counts[a] += 1;
        for (int k = 0; k < d; ++k) sums[(int64_t)a * d + k] += (double)X[i * d + k];
    }
    for (int j = 0; j < C; ++j) {
        if (counts[j] == 0) continue;
        for (int k = 0; k < d; ++k)
            cent[(int64_t)j * d + k] = (float)(sums[(int64_t)j * d + k] / (double)counts[j]);
    }
    free(sums); free(counts);
    return ORC_OK;
}

/* Full k-means: init (or the given centroids), then iters x (assign, update).
 * inertia_hist (optional, length iters) records the inertia of each assign. */
int orc_kmeans(const float* X, int64_t N, int d, int C, int iters, const float* init,
               float* cent, int32_t* assign, double* inertia_hist)
{
    if (C < 1 || N < 1 || d < 1 || iters < 1) return ORC_ERR_ARG;
    if (init) memcpy(cent, init, sizeof(float) * (size_t)C * (size_t)d);
    else orc_kmeans_init(X, N, d, C, cent);
    for (int t = 0; t < iters; ++t) {
        double inertia = 0.0;
        orc_kmeans_assign(X, N, d, cent, C, assign, &inertia);
        if (inertia_hist) inertia_hist[t] = inertia;
        int rc = orc_kmeans_update(X, N, d, assign, C, cent);
        if (rc) return rc;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Semantic permutation [ABS: tokens reordered by cluster; FIG3 (d)].  [reading] stable counting sort by cluster id: cluster j owns
 * the contiguous range [offsets[j], offsets[j+1]); inside it tokens keep
 * ascending original index.  perm[p] = original index at permuted slot p.    */
/* ------------------------------------------------------------------------- */
int orc_permutation(const int32_t* assign, int64_t N, int C, int32_t* perm, int32_t* offsets)
{
    int64_t* cursor = (int64_t*)calloc((size_t)C + 1, sizeof(int64_t));
    if (!cursor) return ORC_ERR_NOMEM;
    for (int64_t i = 0; i < N; ++i) {
        if (assign[i] < 0 || assign[i] >= C) { free(cursor); return ORC_ERR_ARG; }
        cursor[assign[i] + 1] += 1;
    }
    for (int j = 0; j < C; ++j) cursor[j + 1] += cursor[j];
    for (int j = 0; j <= C; ++j) offsets[j] = (int32_t)cursor[j];
    for (int64_t i = 0; i < N; ++i) perm[cursor[assign[i]]++] = (int32_t)i;
    free(cursor);
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* (b) Centroid scores [FIG3 (b)].  S_ij = scale * <cq_i, ck_j>.
 * [reading] the dot product is one fused multiply-add chain in fp32 over
 * k = 0..d-1 starting from +0, then one fp32 multiply by the softmax scale:
 * every step correctly rounded, hence reproducible bit for bit.              */
/* ------------------------------------------------------------------------- */
void orc_scores(const float* cq, int Cq, const float* ck, int Ck, int d, float scale, float* S)
{
    for (int i = 0; i < Cq; ++i)
        for (int j = 0; j < Ck; ++j) {
            float acc = 0.0f;
            for (int k = 0; k < d; ++k)
                acc = fmaf(cq[(int64_t)i * d + k], ck[(int64_t)j * d + k], acc);
            S[(int64_t)i * Ck + j] = acc * scale;
        }
}

/* ------------------------------------------------------------------------- */
/* Integer sampling weight of a skipped key group [ABS: draw probability
 * follows the estimated attention; FIG3 (b),(c)].
 * [reading] the estimated attention of every key of group j, seen from query
 * group i, is exp(S_ij); the group's mass is |K_j| exp(S_ij), so a key's
 * probability is proportional to q_j ~ 2^24 * exp(S_ij - Smax).  It is held
 * as an integer in [1, 2^24] so that every implementation draws the same
 * indices; exp is evaluated as 2^y with y = (S_ij - Smax) * log2(e) split into
 * an integer and a fractional part, and 2^f = e^(f ln 2) by its Taylor series
 * up to degree 6 (Horner, fmaf).  Keys are never given weight 0 (q >= 1), so
 * every skipped key stays reachable and 1/pi stays finite.  Unbiasedness only
 * needs the log-weight to use the q that was sampled from, not an exact exp. */
/* ------------------------------------------------------------------------- */
static float orc_taylor_coef[7];
static int orc_taylor_ready = 0;

static void orc_taylor_init(void)
{
    /* coefficient k = (ln 2)^k / k!, computed in fp64 and rounded once. */
    double term = 1.0;
    for (int k = 0; k <= 6; ++k) {
        orc_taylor_coef[k] = (float)term;
        term = term * M_LN2 / (double)(k + 1);
    }
    orc_taylor_ready = 1;
}

void orc_taylor_coefficients(float* out7)
{
    if (!orc_taylor_ready) orc_taylor_init();
    for (int k = 0; k < 7; ++k) out7[k] = orc_taylor_coef[k];
}

uint32_t orc_group_weight(float s, float smax)
{
    if (!orc_taylor_ready) orc_taylor_init();
    const float log2e = (float)1.4426950408889634; /* log2(e) rounded to fp32 */
    float y = (s - smax) * log2e;
    if (y < -24.0f) return 1u;
    float n = floorf(y);
    float f = y - n;
    float p = orc_taylor_coef[6];
    for (int k = 5; k >= 0; --k) p = fmaf(p, f, orc_taylor_coef[k]);
    float v = floorf(ldexpf(p, 24 + (int)n));
    uint32_t q = (uint32_t)v;
    return q < 1u ? 1u : q;
}

/* ------------------------------------------------------------------------- */
/* (c) Exact set, pi and the group-shared sample for one query group i.
 *
 * Exact set [ABS: the best-scoring keys are attended exactly; FIG3 (c): the
 * first-ranked key group is never dropped].  [reading] non-empty
 * key groups ranked by S_ij descending (ties: lowest j); the rank-0 group is
 * always taken; the next groups are taken while the running key count stays
 * <= E, stopping at the first group that does not fit (a prefix of the
 * ranking).
 *
 * Sample [ABS, FIG3 (c), ICLR].  The skipped keys are the keys of the
 * non-empty groups outside the exact set.  [reading] m draws with replacement,
 * one shared list per query group; draw t uses Philox4x32-10 with key =
 * (seed low, seed high) and counter = (t, i, bh, layer); u = r1*2^32 + r0,
 * r = floor(u * T / 2^64) with T = sum_j |K_j| q_j over skipped groups (j
 * ascending, the CDF order); the group is the first with CDF_j > r and the
 * key offset in it is (r - CDF_{j-1}) / q_j (integer division: uniform inside
 * the group).  The key's probability is p = q_j / T, and its log-weight is
 * log(1/(p m)) = ln T - ln q_j - ln m, which is added to its logit so that
 * the m draws stand for the whole skipped region (ICLR: the weights make the
 * sample represent every skipped key).  No skipped keys -> no draws.
 *
 * Uniform variant (mode 1; Figure 2/4/5 captions run "uniform" sampling):
 * q_j = 1 for every skipped group.
 *
 * Outputs for the group:
 *   exact_groups[0..n_exact)  group ids in rank order (rest set to -1)
 *   counts[0] = n_exact groups, counts[1] = exact keys, counts[2] = draws
 *   sample_pos[0..draws)      permuted key positions, in draw order
 *   sample_bias[0..draws)     log-weights (fp64)
 *   qw[j], cdf info (optional) for the tests
 * ------------------------------------------------------------------------- */
typedef struct {
    int64_t E, m;
    uint64_t seed;
    uint32_t layer, bh;
    int mode; /* 0 importance, 1 uniform */
} orc_select_cfg;

int orc_select_sample_group(const float* S_row, const int32_t* k_offsets, int Ck, int i,
                            const orc_select_cfg* cfg, const int32_t* votes_row /* [Ck] or NULL */,
                            int32_t* exact_groups, int32_t* counts,
                            int32_t* sample_pos, double* sample_bias,
                            uint32_t* qw_out /* [Ck] or NULL: 0 for non-skipped */,
                            uint64_t* total_out /* or NULL */)
{
    int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(Ck > 0 ? Ck : 1));
    uint8_t* in_exact = (uint8_t*)calloc((size_t)(Ck > 0 ? Ck : 1), 1);
    uint32_t* qw = (uint32_t*)calloc((size_t)(Ck > 0 ? Ck : 1), sizeof(uint32_t));
    uint64_t* cdf = (uint64_t*)calloc((size_t)(Ck > 0 ? Ck : 1), sizeof(uint64_t));
    if (!order || !in_exact || !qw || !cdf) { free(order); free(in_exact); free(qw); free(cdf); return ORC_ERR_NOMEM; }

    /* rank the non-empty groups: plain insertion sort, S descending, j
     * ascending; with votes (product-quantised voting), votes descending first */
    int nz = 0;
    for (int j = 0; j < Ck; ++j) {
        if (k_offsets[j + 1] - k_offsets[j] <= 0) continue;
        int pos = nz++;
        while (pos > 0) {
            int prev = order[pos - 1];
            float sp = S_row[prev], sj = S_row[j];
            int before = (sp > sj) || (sp == sj && prev < j);
            if (votes_row && votes_row[prev] != votes_row[j]) before = votes_row[prev] > votes_row[j];
            if (before) break;
            order[pos] = prev;
            --pos;
        }
        order[pos] = j;
    }

    for (int r = 0; r < Ck; ++r) exact_groups[r] = -1;
    int n_exact = 0;
    int64_t exact_keys = 0;
    for (int r = 0; r < nz; ++r) {
        int j = order[r];
        int64_t cnt = k_offsets[j + 1] - k_offsets[j];
        if (r > 0 && exact_keys + cnt > cfg->E) break;
        exact_groups[n_exact++] = j;
        in_exact[j] = 1;
        exact_keys += cnt;
    }

    /* pi over the skipped groups */
    int any_skipped = 0;
    float smax = -INFINITY;
    for (int j = 0; j < Ck; ++j) {
        if (in_exact[j] || k_offsets[j + 1] - k_offsets[j] <= 0) continue;
        if (!any_skipped || S_row[j] > smax) smax = S_row[j];
        any_skipped = 1;
    }
    uint64_t total = 0;
    for (int j = 0; j < Ck; ++j) {
        int64_t cnt = k_offsets[j + 1] - k_offsets[j];
        if (in_exact[j] || cnt <= 0) { cdf[j] = total; continue; }
        qw[j] = (cfg->mode == 1) ? 1u : orc_group_weight(S_row[j], smax);
        total += (uint64_t)cnt * (uint64_t)qw[j];
        cdf[j] = total; /* inclusive */
    }

    int64_t draws = any_skipped ? cfg->m : 0;
    const uint32_t key[2] = { (uint32_t)(cfg->seed & 0xffffffffu), (uint32_t)(cfg->seed >> 32) };
    const double log_total = log((double)total);
    const double log_m = draws > 0 ? log((double)draws) : 0.0;
    for (int64_t t = 0; t < draws; ++t) {
        uint32_t ctr[4] = { (uint32_t)t, (uint32_t)i, cfg->bh, cfg->layer };
        uint32_t rnd[4];
        orc_philox4x32_10(ctr, key, rnd);
        uint64_t u = ((uint64_t)rnd[1] << 32) | (uint64_t)rnd[0];
        uint64_t r = (uint64_t)(((unsigned __int128)u * (unsigned __int128)total) >> 64);
        int jsel = -1;
        for (int j = 0; j < Ck; ++j) {
            if (in_exact[j] || k_offsets[j + 1] - k_offsets[j] <= 0) continue;
            if (cdf[j] > r) { jsel = j; break; }
        }
        if (jsel < 0) { free(order); free(in_exact); free(qw); free(cdf); return ORC_ERR_ARG; }
        uint64_t start = cdf[jsel] - (uint64_t)(k_offsets[jsel + 1] - k_offsets[jsel]) * qw[jsel];
        uint64_t o = (r - start) / qw[jsel];
        sample_pos[t] = k_offsets[jsel] + (int32_t)o;
        sample_bias[t] = log_total - log((double)qw[jsel]) - log_m;
    }

    counts[0] = n_exact;
    counts[1] = (int32_t)exact_keys;
    counts[2] = (int32_t)draws;
    if (qw_out) memcpy(qw_out, qw, sizeof(uint32_t) * (size_t)Ck);
    if (total_out) *total_out = total;
    free(order); free(in_exact); free(qw); free(cdf);
    return ORC_OK;
}

/* Whole head: scores from the given centroids, then every query group.
 * exact_groups [Cq,Ck], counts [Cq,3], sample_pos [Cq,m], sample_bias [Cq,m].
 * Unused sample slots hold position -1 and log-weight 0.                      */
int orc_select_sample(const float* cq, int Cq, const float* ck, int Ck, int d, float scale,
                      const int32_t* k_offsets, const orc_select_cfg* cfg,
                      const int32_t* votes /* [Cq][Ck] or NULL */,
                      int32_t* exact_groups, int32_t* counts,
                      int32_t* sample_pos, double* sample_bias)
{
    float* S = (float*)malloc(sizeof(float) * (size_t)Cq * (size_t)Ck);
    if (!S) return ORC_ERR_NOMEM;
    orc_scores(cq, Cq, ck, Ck, d, scale, S);
    int rc = ORC_OK;
    for (int i = 0; i < Cq && rc == ORC_OK; ++i) {
        int32_t* sp = sample_pos + (int64_t)i * cfg->m;
        double* sb = sample_bias + (int64_t)i * cfg->m;
        for (int64_t t = 0; t < cfg->m; ++t) { sp[t] = -1; sb[t] = 0.0; }
        rc = orc_select_sample_group(S + (int64_t)i * Ck, k_offsets, Ck, i, cfg,
                                     votes ? votes + (int64_t)i * Ck : NULL,
                                     exact_groups + (int64_t)i * Ck, counts + 3 * i,
                                     sp, sb, NULL, NULL);
    }
    free(S);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Top-p key-group selection: the comparator the pages set InstaGen against
 * (thelatestinai.com paper page, Figure 2 caption: SVG2 with Cq = 100,
 * Ck = 500, key floor 0.1, at top-p 0.5 / 0.75 / 0.9 / 0.95; ICLR listing
 * abstract: top-p keeps the highest-scoring blocks and varies their number to
 * reach a target share of the attention mass; the dropped blocks are simply
 * skipped, with no sample).  Every step beyond that sentence is a [reading]:
 *   - estimated attention mass of key group j for query group i: |K_j| times
 *     the per-key estimate exp(S_ij), in the same integer fixed point as the
 *     sampling weights: W_j = |K_j| * q_j with q_j = orc_group_weight(S_ij,
 *     max over all non-empty groups of S_ij), T = sum_j W_j;
 *   - groups ranked by W_j descending (ties: lowest j), the nucleus order;
 *   - the kept set is the shortest prefix of that ranking whose mass reaches
 *     the share p, cum * 2^20 >= p_fix * T with p_fix = round(p * 2^20), and
 *     which holds at least F = round(key_floor * N) keys (the key floor); the
 *     first-ranked group is always kept;
 *   - no draws.
 * Integer arithmetic throughout (T < 2^44 for N < 2^20), so the kept set is
 * reproducible bit for bit.
 * Outputs as orc_select_sample_group: exact_groups in rank order (rest -1),
 * counts = {kept groups, kept keys, 0}; W_out[j] (optional) the masses.      */
/* ------------------------------------------------------------------------- */
int orc_select_top_p_group(const float* S_row, const int32_t* k_offsets, int Ck, float top_p,
                           int64_t floor_keys, int32_t* exact_groups, int32_t* counts,
                           uint64_t* W_out /* [Ck] or NULL */, uint64_t* total_out /* or NULL */)
{
    int32_t* order = (int32_t*)malloc(sizeof(int32_t) * (size_t)(Ck > 0 ? Ck : 1));
    uint64_t* W = (uint64_t*)calloc((size_t)(Ck > 0 ? Ck : 1), sizeof(uint64_t));
    if (!order || !W) { free(order); free(W); return ORC_ERR_NOMEM; }
    const int64_t p_fix = llround((double)top_p * 1048576.0);

    float smax = -INFINITY;
    int any = 0;
    for (int j = 0; j < Ck; ++j) {
        if (k_offsets[j + 1] - k_offsets[j] <= 0) continue;
        if (!any || S_row[j] > smax) smax = S_row[j];
        any = 1;
    }
    uint64_t total = 0;
    for (int j = 0; j < Ck; ++j) {
        const int64_t cnt = k_offsets[j + 1] - k_offsets[j];
        if (cnt <= 0) continue;
        W[j] = (uint64_t)cnt * (uint64_t)orc_group_weight(S_row[j], smax);
        total += W[j];
    }
    /* plain insertion sort: W descending, j ascending */
    int nz = 0;
    for (int j = 0; j < Ck; ++j) {
        if (k_offsets[j + 1] - k_offsets[j] <= 0) continue;
        int pos = nz++;
        while (pos > 0) {
            const int prev = order[pos - 1];
            if (W[prev] > W[j] || (W[prev] == W[j] && prev < j)) break;
            order[pos] = prev;
            --pos;
        }
        order[pos] = j;
    }
    for (int r = 0; r < Ck; ++r) exact_groups[r] = -1;
    uint64_t cum = 0;
    int64_t keys = 0;
    int n = 0;
    for (int r = 0; r < nz; ++r) {
        const int j = order[r];
        exact_groups[n++] = j;
        cum += W[j];
        keys += k_offsets[j + 1] - k_offsets[j];
        if (cum * 1048576ull >= (uint64_t)p_fix * total && keys >= floor_keys) break;
    }
    counts[0] = n;
    counts[1] = (int32_t)keys;
    counts[2] = 0;
    if (W_out) memcpy(W_out, W, sizeof(uint64_t) * (size_t)Ck);
    if (total_out) *total_out = total;
    free(order); free(W);
    return ORC_OK;
}

/* Whole head: scores from the given centroids, then every query group.      */
int orc_select_top_p(const float* cq, int Cq, const float* ck, int Ck, int d, float scale,
                     const int32_t* k_offsets, float top_p, int64_t floor_keys,
                     int32_t* exact_groups, int32_t* counts)
{
    float* S = (float*)malloc(sizeof(float) * (size_t)Cq * (size_t)Ck);
    if (!S) return ORC_ERR_NOMEM;
    orc_scores(cq, Cq, ck, Ck, d, scale, S);
    int rc = ORC_OK;
    for (int i = 0; i < Cq && rc == ORC_OK; ++i)
        rc = orc_select_top_p_group(S + (int64_t)i * Ck, k_offsets, Ck, top_p, floor_keys,
                                    exact_groups + (int64_t)i * Ck, counts + 3 * i, NULL, NULL);
    free(S);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* Product-quantised per-query voting (the selection rule of the abstract:
 * queries and keys are product-quantised so that a block score is cheap for
 * every query, each query votes for its top blocks, and the cluster attends
 * to the most-voted blocks).  The pages fix nothing beyond that sentence;
 * every parameter below is a [reading]:
 *   - subspaces of 8 consecutive dimensions (M = d/8), 16 codewords each, one
 *     codebook per side (queries, keys) and head;
 *   - a codebook is trained by 5 Lloyd iterations on the group centroids of
 *     its side (cq for queries, ck for keys), initialised with the first
 *     min(16, C) of them; distances sum (x_e - c_e)^2 with fmaf over e = 0..7
 *     from +0; ties go to the lowest codeword; a codeword's update is the
 *     fp32 sum of its members in point order divided by their count (fp32);
 *     an empty codeword keeps its value;
 *   - a query token is encoded against the query codebook, a key group by
 *     its centroid against the key codebook (nearest codeword, same rule);
 *   - block score s(q, j) = sum over m = 0..M-1 (fp32 adds from +0) of
 *     T_m[a_m(q)][b_m(j)], T_m[a][b] = the fmaf chain over e of the two
 *     codewords' products;
 *   - query q votes for the prefix of its ranking (non-empty groups by s
 *     descending, ties lowest j) chosen by the exact-set budget rule: rank 0
 *     always, then while the running key count stays <= E;
 *   - the group ranks key groups by votes descending, then by the centroid
 *     score S_ij descending and j ascending, and takes the exact set by the
 *     same budget rule; pi and the sample stay those of the centroid scores.
 * Every decision is a correctly rounded fp32 operation in a fixed order, so
 * an implementation that follows the same order agrees bit for bit.          */
/* ------------------------------------------------------------------------- */
#define ORC_PQ_SUB 8
#define ORC_PQ_KC 16
#define ORC_PQ_ITERS 5

static float orc_pq_dist(const float* x, const float* c)
{
    float acc = 0.0f;
    for (int e = 0; e < ORC_PQ_SUB; ++e) {
        float t = x[e] - c[e];
        acc = fmaf(t, t, acc);
    }
    return acc;
}

/* nearest of kc codewords (cb: kc x 8), ties to the lowest index */
static int orc_pq_nearest(const float* x, const float* cb, int kc)
{
    int best = 0;
    float bd = orc_pq_dist(x, cb);
    for (int c = 1; c < kc; ++c) {
        float dd = orc_pq_dist(x, cb + (size_t)c * ORC_PQ_SUB);
        if (dd < bd) { bd = dd; best = c; }
    }
    return best;
}

/* Codebook of C points P [C, d] (d % 8 == 0): cb [M][16][8] (codewords past
 * min(16, C) are zero and never chosen), codes [C][M] of the points against
 * the final codebook.  Returns the number of codewords in use.               */
int orc_pq_codebook(const float* P, int C, int d, float* cb, uint8_t* codes)
{
    const int M = d / ORC_PQ_SUB;
    const int kc = C < ORC_PQ_KC ? C : ORC_PQ_KC;
    if (C < 1 || d % ORC_PQ_SUB) return -1;
    memset(cb, 0, sizeof(float) * (size_t)M * ORC_PQ_KC * ORC_PQ_SUB);
    int* a = (int*)malloc(sizeof(int) * (size_t)C);
    if (!a) return -1;
    for (int m = 0; m < M; ++m) {
        float* cbm = cb + (size_t)m * ORC_PQ_KC * ORC_PQ_SUB;
        for (int c = 0; c < kc; ++c)
            for (int e = 0; e < ORC_PQ_SUB; ++e) cbm[c * ORC_PQ_SUB + e] = P[(size_t)c * d + m * ORC_PQ_SUB + e];
        for (int it = 0; it < ORC_PQ_ITERS; ++it) {
            for (int p = 0; p < C; ++p) a[p] = orc_pq_nearest(P + (size_t)p * d + m * ORC_PQ_SUB, cbm, kc);
            for (int c = 0; c < kc; ++c) {
                float sum[ORC_PQ_SUB] = {0};
                int n = 0;
                for (int p = 0; p < C; ++p) {
                    if (a[p] != c) continue;
                    for (int e = 0; e < ORC_PQ_SUB; ++e) sum[e] += P[(size_t)p * d + m * ORC_PQ_SUB + e];
                    ++n;
                }
                if (n > 0)
                    for (int e = 0; e < ORC_PQ_SUB; ++e) cbm[c * ORC_PQ_SUB + e] = sum[e] / (float)n;
            }
        }
        if (codes)
            for (int p = 0; p < C; ++p)
                codes[(size_t)p * M + m] = (uint8_t)orc_pq_nearest(P + (size_t)p * d + m * ORC_PQ_SUB, cbm, kc);
    }
    free(a);
    return kc;
}

/* codes [n][M] of the rows X [n, d] against cb (kc codewords in use) */
void orc_pq_encode(const float* X, int64_t n, int d, const float* cb, int kc, uint8_t* codes)
{
    const int M = d / ORC_PQ_SUB;
    for (int64_t p = 0; p < n; ++p)
        for (int m = 0; m < M; ++m)
            codes[p * M + m] = (uint8_t)orc_pq_nearest(X + p * d + m * ORC_PQ_SUB,
                                                       cb + (size_t)m * ORC_PQ_KC * ORC_PQ_SUB, kc);
}

typedef struct { float s; int j; } orc_pq_ranked;

/* ranking order: score descending, then the lower group index */
static int orc_pq_rank_cmp(const void* pa, const void* pb)
{
    const orc_pq_ranked* a = (const orc_pq_ranked*)pa;
    const orc_pq_ranked* b = (const orc_pq_ranked*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

/* Votes of one head: Q [N, d] (original token order), query groups through
 * q_perm / q_offsets, the two codebooks (kcq, kck codewords in use), the key
 * groups' codes kcodes [Ck][M] and k_offsets; votes [Cq][Ck].                */
int orc_pq_votes(const float* Q, int64_t N, int d, const int32_t* q_perm, const int32_t* q_offsets, int Cq,
                 const float* cbq, int kcq, const float* cbk, int kck, const uint8_t* kcodes,
                 const int32_t* k_offsets, int Ck, int64_t E, int32_t* votes)
{
    const int M = d / ORC_PQ_SUB;
    float* T = (float*)malloc(sizeof(float) * (size_t)M * ORC_PQ_KC * ORC_PQ_KC);
    orc_pq_ranked* order = (orc_pq_ranked*)malloc(sizeof(orc_pq_ranked) * (size_t)(Ck > 0 ? Ck : 1));
    uint8_t* qc = (uint8_t*)malloc((size_t)M);
    if (!T || !order || !qc) { free(T); free(order); free(qc); return ORC_ERR_NOMEM; }
    for (int m = 0; m < M; ++m)
        for (int a = 0; a < ORC_PQ_KC; ++a)
            for (int b = 0; b < ORC_PQ_KC; ++b) {
                const float* x = cbq + ((size_t)m * ORC_PQ_KC + a) * ORC_PQ_SUB;
                const float* y = cbk + ((size_t)m * ORC_PQ_KC + b) * ORC_PQ_SUB;
                float acc = 0.0f;
                for (int e = 0; e < ORC_PQ_SUB; ++e) acc = fmaf(x[e], y[e], acc);
                T[((size_t)m * ORC_PQ_KC + a) * ORC_PQ_KC + b] = acc;
            }
    memset(votes, 0, sizeof(int32_t) * (size_t)Cq * (size_t)Ck);
    int rc = ORC_OK;
    for (int i = 0; i < Cq && rc == ORC_OK; ++i) {
        for (int64_t slot = q_offsets[i]; slot < q_offsets[i + 1]; ++slot) {
            const int64_t q = q_perm[slot];
            if (q < 0 || q >= N) { rc = ORC_ERR_ARG; break; }
            orc_pq_encode(Q + q * d, 1, d, cbq, kcq, qc);
            int nz = 0;
            for (int j = 0; j < Ck; ++j) {
                if (k_offsets[j + 1] - k_offsets[j] <= 0) continue;
                float acc = 0.0f;
                for (int m = 0; m < M; ++m)
                    acc += T[((size_t)m * ORC_PQ_KC + qc[m]) * ORC_PQ_KC + kcodes[(size_t)j * M + m]];
                order[nz].s = acc;
                order[nz].j = j;
                ++nz;
            }
            qsort(order, (size_t)nz, sizeof(orc_pq_ranked), orc_pq_rank_cmp);
            int64_t keys = 0;
            for (int r = 0; r < nz; ++r) {
                const int j = order[r].j;
                const int64_t cnt = k_offsets[j + 1] - k_offsets[j];
                if (r > 0 && keys + cnt > E) break;
                keys += cnt;
                votes[(int64_t)i * Ck + j] += 1;
            }
        }
    }
    (void)kck;
    free(T); free(order); free(qc);
    return rc;
}

/* ------------------------------------------------------------------------- */
/* (d) Attention over the exact keys plus the weighted sample [ABS, FIG3 (d),
 * ICLR].  For query q (original index) in group i = q_assign[q]:
 *   keys   = every key of the exact groups (original index k_perm[p] for p in
 *            [k_off[g], k_off[g+1])) and every sample slot t (original index
 *            k_perm[sample_pos[i][t]]), a key drawn twice counting twice;
 *   logit  = scale * <q, k>  (+ sample_bias[i][t] for slot t);
 *   out    = sum softmax(logit) * v, all in fp64.
 * rows lists the original query indices to compute; out is [nrows, d].      */
/* ------------------------------------------------------------------------- */
int orc_attention_rows(const float* Q, const float* K, const float* V, int64_t N, int d, float scale,
                       const int32_t* q_assign, const int32_t* k_perm, const int32_t* k_offsets, int Ck,
                       const int32_t* exact_groups, const int32_t* counts,
                       const int32_t* sample_pos, const double* sample_bias, int64_t m_stride,
                       const int64_t* rows, int64_t nrows, double* out)
{
    int bad = 0;
    #pragma omp parallel for schedule(dynamic, 4) reduction(|:bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t q = rows[r];
        double* o = out + r * d;
        for (int k = 0; k < d; ++k) o[k] = 0.0;
        if (q < 0 || q >= N) { bad |= 1; continue; }
        int i = q_assign[q];
        const float* qv = Q + q * d;
        int ne = counts[3 * i + 0], ns = counts[3 * i + 2];
        /* pass 1: maximum logit */
        double mx = -INFINITY;
        for (int e = 0; e < ne; ++e) {
            int g = exact_groups[(int64_t)i * Ck + e];
            for (int32_t p = k_offsets[g]; p < k_offsets[g + 1]; ++p) {
                const float* kv = K + (int64_t)k_perm[p] * d;
                double s = 0.0;
                for (int k = 0; k < d; ++k) s += (double)qv[k] * (double)kv[k];
                s *= (double)scale;
                if (s > mx) mx = s;
            }
        }
        for (int t = 0; t < ns; ++t) {
            int32_t p = sample_pos[(int64_t)i * m_stride + t];
            const float* kv = K + (int64_t)k_perm[p] * d;
            double s = 0.0;
            for (int k = 0; k < d; ++k) s += (double)qv[k] * (double)kv[k];
            s = s * (double)scale + sample_bias[(int64_t)i * m_stride + t];
            if (s > mx) mx = s;
        }
        /* pass 2: weights and the weighted sum of values */
        double den = 0.0;
        for (int e = 0; e < ne; ++e) {
            int g = exact_groups[(int64_t)i * Ck + e];
            for (int32_t p = k_offsets[g]; p < k_offsets[g + 1]; ++p) {
                int64_t kk = k_perm[p];
                const float* kv = K + kk * d;
                double s = 0.0;
                for (int k = 0; k < d; ++k) s += (double)qv[k] * (double)kv[k];
                double w = exp(s * (double)scale - mx);
                den += w;
                for (int k = 0; k < d; ++k) o[k] += w * (double)V[kk * d + k];
            }
        }
        for (int t = 0; t < ns; ++t) {
            int32_t p = sample_pos[(int64_t)i * m_stride + t];
            int64_t kk = k_perm[p];
            const float* kv = K + kk * d;
            double s = 0.0;
            for (int k = 0; k < d; ++k) s += (double)qv[k] * (double)kv[k];
            double w = exp(s * (double)scale + sample_bias[(int64_t)i * m_stride + t] - mx);
            den += w;
            for (int k = 0; k < d; ++k) o[k] += w * (double)V[kk * d + k];
        }
        for (int k = 0; k < d; ++k) o[k] /= den;
    }
    return bad ? ORC_ERR_ARG : ORC_OK;
}

/* Threads an OpenMP parallel region of the oracle uses (for reporting). */
#ifdef _OPENMP
#include <omp.h>
#endif
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
