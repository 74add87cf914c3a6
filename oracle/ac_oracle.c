/*
 * ac_oracle.c -- CPU oracle of the cluster-routed sparse attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * product never links, imports or calls it, and shares no code with it.
 *
 * It is a plain, slow, step-by-step restatement of the method on the page
 * "AdaCluster: Adaptive Query-Key Clustering for Sparse Attention in Video
 * Generation" (arXiv 2604.18348):
 *   - Sec. 3.1 and App. A.2: queries are L2-normalised, then clustered with
 *     standard k-means (angular clustering);
 *   - Sec. 3.2.2, Algorithm 1 (MultiStageClustering): keys are clustered in
 *     stages, outliers (distance to centre >= tau) are re-clustered, and a
 *     head whose cluster count reaches N_max falls back to dense attention;
 *   - Sec. 3.2.1: per-head MSE and compactness Comp = 1/MSE;
 *   - Sec. 3.2.3, Eq. (1) and Algorithm 2 (TensorQuest): the Quest upper bound
 *     sum_d max(q_d max K_d, q_d min K_d) scores every key cluster;
 *   - Algorithm 3 (AdaCluster): top-k key clusters per query cluster, then
 *     exact softmax attention over the tokens of the selected clusters.
 *
 * Precision: the clustering, removal, scoring and selection decisions are
 * taken in fp32 with a fixed, sequential operation order (the precision the
 * kernels decide in).  Attention is evaluated in fp64 (its definition).
 * Build with -ffp-contract=off so that no multiply-add is fused.
 *
 * Readings of points the pages leave open are stated at each function.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_TAU_ABSOLUTE 0
#define OR_TAU_MEAN_FACTOR 1
#define OR_TAU_PERCENTILE 2

typedef struct or_cfg {
    int Cq;          /* query clusters (65 on the pages, Sec. 4.1) */
    int m0;          /* initial key cluster count of stage 0 */
    int n_max;       /* N_max of Algorithm 1 */
    int tau_mode;    /* OR_TAU_* */
    float tau_value; /* absolute tau / factor of the mean / permille */
    int topk;        /* >0: clusters per query cluster; <0: -permille of n_k */
    int iters_q;     /* Lloyd iterations for queries */
    int iters_k;     /* Lloyd iterations per key stage */
    int iters_warm;  /* Lloyd iterations in a warm-started step */
    int stage_rule;  /* cluster count of stages t > 0, see or_stage_clusters */
    uint64_t seed;
    int64_t unit0;   /* (batch, head) index of the first unit of the call: unit h of
                        the call draws its initial centres as unit unit0 + h, so a
                        head can be run on its own with the seeds of the whole layer */
} or_cfg;

/* ------------------------------------------------------------------ */
/* helpers                                                              */
/* ------------------------------------------------------------------ */

static float bf2f(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* SplitMix64 output function (Steele, Lea, Flood: "Fast splittable
 * pseudorandom number generators", OOPSLA 2014). */
static uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

#define OR_GAMMA 0x9E3779B97F4A7C15ull

/* The (i+1)-th output of SplitMix64 started from `state`. */
uint64_t or_splitmix64(uint64_t state, int64_t i)
{
    return mix64(state + (uint64_t)(i + 1) * OR_GAMMA);
}

/* Counter-based stream: the (i+1)-th SplitMix64 output of a generator keyed
 * by (seed, bh, tag). */
uint64_t or_rand(uint64_t seed, int64_t bh, int32_t tag, int64_t i)
{
    uint64_t key = mix64(seed ^ mix64((((uint64_t)bh) << 32) ^ (uint64_t)(uint32_t)tag));
    return or_splitmix64(key, i);
}

/* Seeded initial centres.  The pages only say "standard KMeans" (Sec. 3.3)
 * and "a moderate cluster number" (Algorithm 1); the initialisation is not
 * given.  Reading: a seeded, Forgy-style sample of m distinct members of the
 * set being clustered (members in ascending token order, n of them).  Centre
 * j is member pos[j], drawn uniformly from the j-th of m equal strata
 * [floor(j n / m), floor((j+1) n / m)).  Requires 1 <= m <= n. */
void or_seed_pick(uint64_t seed, int64_t bh, int32_t tag, int64_t n, int32_t m, int64_t *pos)
{
    for (int32_t j = 0; j < m; ++j) {
        int64_t lo = ((int64_t)j * n) / m;
        int64_t hi = ((int64_t)(j + 1) * n) / m;
        pos[j] = lo + (int64_t)(or_rand(seed, bh, tag, j) % (uint64_t)(hi - lo));
    }
}

/* Squared Euclidean distance, summed over dimensions in index order. */
static float sqdist(const float *x, const float *c, int d)
{
    float s = 0.0f;
    for (int k = 0; k < d; ++k) {
        float t = x[k] - c[k];
        s = s + t * t;
    }
    return s;
}

/* ------------------------------------------------------------------ */
/* Sec. 3.1: query normalisation                                        */
/* ------------------------------------------------------------------ */

/* inv[i] = 1/||q_i||_2 and xhat = q * inv.  Reading: the normalised query is
 * kept in fp32.  A zero query has no direction; reading: its xhat is 0. */
void or_qnorm(const uint16_t *Q, int64_t rows, int d, float *inv, float *xhat)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
        const uint16_t *q = Q + i * d;
        float ss = 0.0f;
        for (int k = 0; k < d; ++k) {
            float v = bf2f(q[k]);
            ss = ss + v * v;
        }
        float r = (ss > 0.0f) ? 1.0f / sqrtf(ss) : 0.0f;
        if (inv) inv[i] = r;
        if (xhat)
            for (int k = 0; k < d; ++k) xhat[i * d + k] = bf2f(q[k]) * r;
    }
}

/* ------------------------------------------------------------------ */
/* Lloyd's k-means ("standard KMeans", Sec. 3.3)                        */
/* ------------------------------------------------------------------ */

/* Assignment: label = argmin_c ||x - c||^2, exact ties to the lowest c;
 * dmin receives the winning squared distance. */
void or_assign(const float *X, int64_t n, int d, const float *C, int m,
               int32_t *labels, float *dmin)
{
#pragma omp parallel for schedule(static) if (n > 4096)
    for (int64_t i = 0; i < n; ++i) {
        const float *x = X + i * d;
        float best = INFINITY;
        int32_t arg = 0;
        for (int c = 0; c < m; ++c) {
            float v = sqdist(x, C + (int64_t)c * d, d);
            if (v < best) {
                best = v;
                arg = c;
            }
        }
        labels[i] = arg;
        if (dmin) dmin[i] = best;
    }
}

/* Update: each centre becomes the mean of its members, the members summed in
 * ascending order in fp32 and the sum divided by the count.  Reading: an
 * empty cluster keeps its previous centre.  counts may be NULL. */
void or_update(const float *X, int64_t n, int d, const int32_t *labels, int m,
               float *C, int32_t *counts)
{
    float *sum = (float *)calloc((size_t)m * d, sizeof(float));
    int64_t *cnt = (int64_t *)calloc((size_t)m, sizeof(int64_t));
    for (int64_t i = 0; i < n; ++i) {
        int32_t c = labels[i];
        cnt[c] += 1;
        for (int k = 0; k < d; ++k) sum[(int64_t)c * d + k] = sum[(int64_t)c * d + k] + X[i * d + k];
    }
    for (int c = 0; c < m; ++c) {
        if (cnt[c] > 0) {
            float fc = (float)cnt[c];
            for (int k = 0; k < d; ++k) C[(int64_t)c * d + k] = sum[(int64_t)c * d + k] / fc;
        }
        if (counts) counts[c] = (int32_t)cnt[c];
    }
    free(sum);
    free(cnt);
}

/* Objective J = sum_i ||x_i - C[labels_i]||^2 in fp64 (self-check only). */
double or_objective(const float *X, int64_t n, int d, const float *C, const int32_t *labels)
{
    double J = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        const float *x = X + i * d;
        const float *c = C + (int64_t)labels[i] * d;
        for (int k = 0; k < d; ++k) {
            double t = (double)x[k] - (double)c[k];
            J += t * t;
        }
    }
    return J;
}

/* T Lloyd iterations (assign, update) from the centres in C, then one final
 * assignment, whose labels and distances are returned.  The iteration count
 * is not on the pages; reading: fixed counts given by the caller.
 * jtrace (nullable, 2T+1 entries) receives J after every half-step. */
void or_kmeans(const float *X, int64_t n, int d, float *C, int m, int T,
               int32_t *labels, float *dmin, double *jtrace)
{
    for (int t = 0; t < T; ++t) {
        or_assign(X, n, d, C, m, labels, NULL);
        if (jtrace) jtrace[2 * t] = or_objective(X, n, d, C, labels);
        or_update(X, n, d, labels, m, C, NULL);
        if (jtrace) jtrace[2 * t + 1] = or_objective(X, n, d, C, labels);
    }
    or_assign(X, n, d, C, m, labels, dmin);
    if (jtrace) jtrace[2 * T] = or_objective(X, n, d, C, labels);
}

/* ------------------------------------------------------------------ */
/* Algorithm 3 line 3: A_q, C_q <- KMeans(Normalize(Q))                 */
/* ------------------------------------------------------------------ */

/* Q: [BH, L, d] bf16.  init (nullable): [BH, Cq, d] centres of the previous
 * denoising step (warm start, Sec. 3.2.2 "Efficient initialization" and
 * Sec. 4.1: centres of the previous step are reused); otherwise seeded
 * members (tag 0).  Reading: centres stay plain means of unit vectors, they
 * are not renormalised (standard, not spherical, k-means). */
void or_cluster_q(const uint16_t *Q, int BH, int L, int d, const or_cfg *cfg,
                  const float *init, int T, int32_t *labels, float *C, int32_t *counts)
{
    int m = cfg->Cq;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < BH; ++h) {
        float *X = (float *)malloc((size_t)L * d * sizeof(float));
        or_qnorm(Q + (int64_t)h * L * d, L, d, NULL, X);
        float *Ch = C + (int64_t)h * m * d;
        if (init) {
            memcpy(Ch, init + (int64_t)h * m * d, (size_t)m * d * sizeof(float));
        } else {
            int64_t *pos = (int64_t *)malloc((size_t)m * sizeof(int64_t));
            or_seed_pick(cfg->seed, cfg->unit0 + h, 0, L, m, pos);
            for (int j = 0; j < m; ++j) memcpy(Ch + (int64_t)j * d, X + pos[j] * d, (size_t)d * sizeof(float));
            free(pos);
        }
        int32_t *lab = labels + (int64_t)h * L;
        or_kmeans(X, L, d, Ch, m, T, lab, NULL, NULL);
        if (counts) {
            int32_t *cn = counts + (int64_t)h * m;
            memset(cn, 0, (size_t)m * sizeof(int32_t));
            for (int i = 0; i < L; ++i) cn[lab[i]] += 1;
        }
        free(X);
    }
}

/* ------------------------------------------------------------------ */
/* tau (Sec. 4.1 and App. A.5)                                          */
/* ------------------------------------------------------------------ */

static int cmp_float(const void *a, const void *b)
{
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

/* The pages give tau as 1.5x "the average token-to-cluster-center distance
 * computed in the first inference step" (Sec. 4.1) and, in App. A.5, as
 * absolute thresholds.  Reading: one tau per call, computed from the stage-0
 * distances of all heads together (dist, n values).
 *  - mean rule: tau = factor * mean.  The mean is formed from an exact,
 *    order-independent sum of floor(d_i * 2^24) (fixed point, 2^-24 grid),
 *    in integer arithmetic, divided in fp64, then rounded to fp32.
 *  - percentile rule: nearest rank, tau = sorted[ceil(p n / 1000) - 1] with p
 *    in permille.
 *  - absolute rule: tau = value. */
float or_tau(const float *dist, int64_t n, int mode, float value)
{
    if (mode == OR_TAU_ABSOLUTE || n <= 0) return value;
    if (mode == OR_TAU_MEAN_FACTOR) {
        uint64_t s = 0;
        for (int64_t i = 0; i < n; ++i) s += (uint64_t)((double)dist[i] * 16777216.0);
        double mean = ((double)s / 16777216.0) / (double)n;
        return (float)((double)value * mean);
    }
    float *tmp = (float *)malloc((size_t)n * sizeof(float));
    memcpy(tmp, dist, (size_t)n * sizeof(float));
    qsort(tmp, (size_t)n, sizeof(float), cmp_float);
    int64_t p = (int64_t)value;
    int64_t idx = (p * n + 999) / 1000 - 1;
    if (idx < 0) idx = 0;
    if (idx > n - 1) idx = n - 1;
    float t = tmp[idx];
    free(tmp);
    return t;
}

/* ------------------------------------------------------------------ */
/* Algorithm 1: MultiStageClustering                                    */
/* ------------------------------------------------------------------ */

/* Cluster count m_t of stage t (Algorithm 1 line 11, "choose a moderate
 * cluster number m_t"; the prose of Sec. 3.2.2 re-clusters the outliers "with
 * a few number of new clusters").  Readings:
 *   rule 0 (default): every stage makes the same moderate choice as stage 0,
 *     m_t = min(m0, |U|);
 *   rule 1: proportional to what is left, so that the mean cluster size stays
 *     L/m0: m_t = min(|U|, max(1, ceil(m0 |U| / L))). */
int32_t or_stage_clusters(int32_t m0, int64_t nU, int64_t L, int t, int rule)
{
    if (t == 0 || rule == 0) return (int32_t)(m0 < nU ? m0 : nU);
    int64_t m = (m0 * nU + L - 1) / L;
    if (m < 1) m = 1;
    if (m > nU) m = nU;
    return (int32_t)m;
}

/* One stage on the unabsorbed set U (uidx: ascending token indices, nU of
 * them): seeded init (tag 1 + t), T Lloyd iterations, final assignment;
 * dist[j] = sqrt of the winning squared distance of member j.  Centres are
 * written to Ct ([m, d]). */
static void ms_stage(const float *Kf, int d, const int64_t *uidx, int64_t nU, int32_t m,
                     const or_cfg *cfg, int64_t bh, int t, float *Ct, float *dist)
{
    float *X = (float *)malloc((size_t)nU * d * sizeof(float));
    for (int64_t j = 0; j < nU; ++j) memcpy(X + j * d, Kf + uidx[j] * d, (size_t)d * sizeof(float));
    int64_t *pos = (int64_t *)malloc((size_t)m * sizeof(int64_t));
    or_seed_pick(cfg->seed, bh, 1 + t, nU, m, pos);
    for (int j = 0; j < m; ++j) memcpy(Ct + (int64_t)j * d, X + pos[j] * d, (size_t)d * sizeof(float));
    int32_t *lab = (int32_t *)malloc((size_t)nU * sizeof(int32_t));
    float *dm = (float *)malloc((size_t)nU * sizeof(float));
    or_kmeans(X, nU, d, Ct, m, cfg->iters_k, lab, dm, NULL);
    for (int64_t j = 0; j < nU; ++j) dist[j] = sqrtf(dm[j]);
    free(X);
    free(pos);
    free(lab);
    free(dm);
}

/* K: [BH, L, d] bf16.  Outputs:
 *   labels [BH, L]: final assignment to the nearest of all centres (Alg. 1
 *     line 22), ties to the lowest global id; ids are stage-major;
 *   C [BH, Ccap, d] with Ccap = n_max + m0: the centres, not recomputed after
 *     the final assignment (line 23 returns C as is);
 *   n_k [BH], F [BH] (dense fallback), stages [BH], *tau_out;
 *   removed_stage [BH, L] (nullable): the stage at which the token left U
 *     (-1: never), removed_dist [BH, L] (nullable): its distance then.
 * Readings (garbles on the page): "U <- D" (line 4) is U <- K; the removal
 * loop "for each k_i in K" (line 13) runs over the members of U, the only
 * tokens clustered in the stage; removal uses the strict test d_i < tau
 * (line 15); the N_max test sits at the loop head (line 7), so |C| may end
 * above N_max when U empties in the same stage, with F false.  The fallback
 * flag is per (batch, head).  Returns 0, or -1 on invalid arguments. */
int or_cluster_k_multistage(const uint16_t *K, int BH, int L, int d, const or_cfg *cfg,
                            int32_t *labels, float *C, int32_t *n_k, uint8_t *F,
                            float *tau_out, int32_t *stages, int32_t *removed_stage,
                            float *removed_dist)
{
    if (cfg->n_max < 1 || cfg->m0 < 1 || L < 1) return -1;
    const int Ccap = cfg->n_max + cfg->m0;
    float *dist0 = (float *)malloc((size_t)BH * L * sizeof(float));

    /* stage 0 of every head: U = all tokens */
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < BH; ++h) {
        float *Kf = (float *)malloc((size_t)L * d * sizeof(float));
        for (int64_t i = 0; i < (int64_t)L * d; ++i) Kf[i] = bf2f(K[(int64_t)h * L * d + i]);
        int64_t *uidx = (int64_t *)malloc((size_t)L * sizeof(int64_t));
        for (int64_t i = 0; i < L; ++i) uidx[i] = i;
        int32_t m = or_stage_clusters(cfg->m0, L, L, 0, cfg->stage_rule);
        ms_stage(Kf, d, uidx, L, m, cfg, cfg->unit0 + h, 0, C + (int64_t)h * Ccap * d, dist0 + (int64_t)h * L);
        n_k[h] = m;
        free(Kf);
        free(uidx);
    }

    float tau = or_tau(dist0, (int64_t)BH * L, cfg->tau_mode, cfg->tau_value);
    if (tau_out) *tau_out = tau;

#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < BH; ++h) {
        float *Kf = (float *)malloc((size_t)L * d * sizeof(float));
        for (int64_t i = 0; i < (int64_t)L * d; ++i) Kf[i] = bf2f(K[(int64_t)h * L * d + i]);
        int64_t *uidx = (int64_t *)malloc((size_t)L * sizeof(int64_t));
        float *dist = (float *)malloc((size_t)L * sizeof(float));
        int32_t *rs = removed_stage ? removed_stage + (int64_t)h * L : NULL;
        float *rd = removed_dist ? removed_dist + (int64_t)h * L : NULL;
        if (rs)
            for (int i = 0; i < L; ++i) rs[i] = -1;
        float *Ch = C + (int64_t)h * Ccap * d;

        /* stage 0 removal (lines 13-18) */
        int64_t nU = 0;
        for (int64_t i = 0; i < L; ++i) {
            float di = dist0[(int64_t)h * L + i];
            if (di < tau) {
                if (rs) rs[i] = 0;
                if (rd) rd[i] = di;
            } else {
                uidx[nU++] = i;
            }
        }
        int32_t nc = n_k[h];
        uint8_t f = 0;
        int t = 1;
        while (nU > 0) {                 /* line 6 */
            if (nc >= cfg->n_max) {      /* lines 7-9 */
                f = 1;
                break;
            }
            int32_t m = or_stage_clusters(cfg->m0, nU, L, t, cfg->stage_rule); /* line 11 */
            ms_stage(Kf, d, uidx, nU, m, cfg, cfg->unit0 + h, t, Ch + (int64_t)nc * d, dist); /* line 12, 14 */
            int64_t keep = 0;
            for (int64_t j = 0; j < nU; ++j) {                     /* lines 13-18 */
                if (dist[j] < tau) {
                    if (rs) rs[uidx[j]] = t;
                    if (rd) rd[uidx[j]] = dist[j];
                } else {
                    uidx[keep++] = uidx[j];
                }
            }
            nU = keep;
            nc += m;                                               /* line 19 */
            ++t;                                                   /* line 20 */
        }
        n_k[h] = nc;
        F[h] = f;
        if (stages) stages[h] = t;
        /* line 22: every key to its closest centre among all of C */
        or_assign(Kf, L, d, Ch, nc, labels + (int64_t)h * L, NULL);
        free(Kf);
        free(uidx);
        free(dist);
    }
    free(dist0);
    return 0;
}

/* Warm-started step (Sec. 3.2.2 "Efficient initialization"): the cluster
 * count n_k found at the first denoising step is kept, the previous centres
 * are the initial centres, and T Lloyd iterations run over all keys of the
 * head.  Heads with F set stay dense and are skipped. */
void or_cluster_k_warm(const uint16_t *K, int BH, int L, int d, int Ccap, const int32_t *n_k,
                       const uint8_t *F, int T, float *C, int32_t *labels)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < BH; ++h) {
        if (F[h]) continue;
        float *Kf = (float *)malloc((size_t)L * d * sizeof(float));
        for (int64_t i = 0; i < (int64_t)L * d; ++i) Kf[i] = bf2f(K[(int64_t)h * L * d + i]);
        or_kmeans(Kf, L, d, C + (int64_t)h * Ccap * d, n_k[h], T, labels + (int64_t)h * L, NULL, NULL);
        free(Kf);
    }
}

/* ------------------------------------------------------------------ */
/* Sec. 3.2.1 compactness and the per-cluster bounds used by Eq. (1)    */
/* ------------------------------------------------------------------ */

/* Per key cluster: count, per-dimension max and min of the members (exact
 * bf16 values), SSE = sum of squared distances to the centre (members in
 * ascending order, fp32).  Per head: MSE = (sum over clusters of SSE, in
 * cluster order, fp32) / L and Comp = 1 / MSE.  The page writes the MSE with
 * an overloaded index i; reading: the mean over the L keys of one head.
 * Empty clusters get count 0 and max = min = 0. */
void or_key_stats(const uint16_t *K, int BH, int L, int d, int Ccap, const int32_t *n_k,
                  const int32_t *labels, const float *C, int32_t *counts, float *kmax,
                  float *kmin, float *sse, float *mse_out, float *comp)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < BH; ++h) {
        int m = n_k[h];
        int32_t *cn = counts + (int64_t)h * Ccap;
        float *mx = kmax + (int64_t)h * Ccap * d;
        float *mn = kmin + (int64_t)h * Ccap * d;
        float *se = sse + (int64_t)h * Ccap;
        const float *Ch = C + (int64_t)h * Ccap * d;
        for (int c = 0; c < Ccap; ++c) {
            cn[c] = 0;
            se[c] = 0.0f;
            for (int k = 0; k < d; ++k) mx[(int64_t)c * d + k] = mn[(int64_t)c * d + k] = 0.0f;
        }
        float *x = (float *)malloc((size_t)d * sizeof(float));
        for (int64_t i = 0; i < L; ++i) {
            int c = labels[(int64_t)h * L + i];
            for (int k = 0; k < d; ++k) x[k] = bf2f(K[((int64_t)h * L + i) * d + k]);
            for (int k = 0; k < d; ++k) {
                float *a = mx + (int64_t)c * d + k, *b = mn + (int64_t)c * d + k;
                if (cn[c] == 0) {
                    *a = x[k];
                    *b = x[k];
                } else {
                    if (x[k] > *a) *a = x[k];
                    if (x[k] < *b) *b = x[k];
                }
            }
            se[c] = se[c] + sqdist(x, Ch + (int64_t)c * d, d);
            cn[c] += 1;
        }
        free(x);
        float tot = 0.0f;
        for (int c = 0; c < m; ++c) tot = tot + se[c];
        float mse = tot / (float)L;
        if (mse_out) mse_out[h] = mse;
        comp[h] = 1.0f / mse;
    }
}

/* ------------------------------------------------------------------ */
/* Sec. 3.2.3 Eq. (1), Algorithm 2, Algorithm 3 line 9                  */
/* ------------------------------------------------------------------ */

/* S[qc, kc] = sum_d max(q_d * Kmax_d, q_d * Kmin_d) with q the centre of the
 * query cluster (Eq. (1)), summed over d in order in fp32.  Algorithm 2
 * prints its output as [B, H, Lq, Lk]; reading: it is taken per query
 * cluster (Algorithm 3 applies it after query clustering).  Eq. (2) as
 * printed, with k+ = max(k, 0) and k- = min(k, 0), differs from Eq. (1) when
 * max K_d < 0 or min K_d > 0; reading: Eq. (1), the definition.  Empty key
 * clusters score -inf. */
void or_quest(const float *qc, int nq, int d, const float *kmax, const float *kmin,
              const int32_t *counts, int nk, float *S)
{
    for (int a = 0; a < nq; ++a) {
        const float *q = qc + (int64_t)a * d;
        for (int c = 0; c < nk; ++c) {
            if (counts[c] == 0) {
                S[(int64_t)a * nk + c] = -INFINITY;
                continue;
            }
            float s = 0.0f;
            for (int k = 0; k < d; ++k) {
                float u = q[k] * kmax[(int64_t)c * d + k];
                float v = q[k] * kmin[(int64_t)c * d + k];
                s = s + (u > v ? u : v);
            }
            S[(int64_t)a * nk + c] = s;
        }
    }
}

/* The mean-based baseline of the TensorQuest ablation (Sec. 4.4, Table 4,
 * "w/o Quest"): S[qc, kc] = sum_d q_d * mu_d with mu the centre (mean) of the
 * key cluster, summed over d in order in fp32; empty clusters -inf.  Reading:
 * "mean-based" scores the cluster by its centre in place of the Eq. (1) bound. */
void or_mean_scores(const float *qc, int nq, int d, const float *cent, const int32_t *counts, int nk,
                    float *S)
{
    for (int a = 0; a < nq; ++a) {
        const float *q = qc + (int64_t)a * d;
        for (int c = 0; c < nk; ++c) {
            if (counts[c] == 0) {
                S[(int64_t)a * nk + c] = -INFINITY;
                continue;
            }
            float s = 0.0f;
            for (int k = 0; k < d; ++k) s = s + q[k] * cent[(int64_t)c * d + k];
            S[(int64_t)a * nk + c] = s;
        }
    }
}

/* How many key clusters each query cluster keeps.  The pages give "TopK 64"
 * (App. A.5) with no rounding rule.  Reading: topk > 0 is a count; topk < 0
 * is -permille of n_k, k = ceil(permille * n_k / 1000); the result is clamped
 * to [1, number of non-empty clusters]. */
int32_t or_topk_count(int32_t topk, int32_t nk, int32_t nonempty)
{
    int64_t k = topk > 0 ? topk : ((int64_t)(-topk) * nk + 999) / 1000;
    if (k > nonempty) k = nonempty;
    if (k < 1) k = 1;
    return (int32_t)k;
}

static int cmp_score(const void *a, const void *b, void *row)
{
    const float *S = (const float *)row;
    int32_t i = *(const int32_t *)a, j = *(const int32_t *)b;
    float x = S[i], y = S[j];
    if (x > y) return -1;
    if (x < y) return 1;
    return (i > j) - (i < j);
}

/* Index <- argtopk(S, topk): per query cluster, the k highest scores among
 * the non-empty key clusters; ties go to the lower cluster id; the selected
 * ids are returned in ascending id order.  sel: [nq, k]. */
void or_topk(const float *S, int nq, int nk, int32_t k, int32_t *sel)
{
    int32_t *idx = (int32_t *)malloc((size_t)nk * sizeof(int32_t));
    for (int a = 0; a < nq; ++a) {
        for (int c = 0; c < nk; ++c) idx[c] = c;
        qsort_r(idx, (size_t)nk, sizeof(int32_t), cmp_score, (void *)(S + (int64_t)a * nk));
        /* ascending id order of the chosen k */
        char *take = (char *)calloc((size_t)nk, 1);
        for (int j = 0; j < k; ++j) take[idx[j]] = 1;
        int w = 0;
        for (int c = 0; c < nk; ++c)
            if (take[c]) sel[(int64_t)a * k + w++] = c;
        free(take);
    }
    free(idx);
}

/* ------------------------------------------------------------------ */
/* Algorithm 3 lines 5-11: attention                                    */
/* ------------------------------------------------------------------ */

/* For the listed query rows of one head: the key set of query i is the union
 * of the members of the clusters sel[labels_q[i], 0..k) (all keys when dense
 * is set), and o_i = softmax(scale * q_i . k_j) v_j over that set, in fp64
 * with the maximum subtracted.  The scale is not stated; reading: 1/sqrt(d),
 * passed in.  Q, K, V: [L, d] bf16 of one head.  out: [nrows, d]. */
void or_attention_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int L, int d,
                       const int32_t *labels_q, const int32_t *labels_k, const int32_t *sel,
                       int32_t k, int dense, double scale, const int64_t *rows, int64_t nrows,
                       double *out)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows[r];
        double *s = (double *)malloc((size_t)L * sizeof(double));
        char *use = (char *)malloc((size_t)L);
        double *q = (double *)malloc((size_t)d * sizeof(double));
        for (int t = 0; t < d; ++t) q[t] = (double)bf2f(Q[i * d + t]);
        if (dense) {
            memset(use, 1, (size_t)L);
        } else {
            memset(use, 0, (size_t)L);
            const int32_t *my = sel + (int64_t)labels_q[i] * k;
            for (int64_t j = 0; j < L; ++j)
                for (int a = 0; a < k; ++a)
                    if (labels_k[j] == my[a]) {
                        use[j] = 1;
                        break;
                    }
        }
        double mx = -INFINITY;
        for (int64_t j = 0; j < L; ++j) {
            if (!use[j]) continue;
            double acc = 0.0;
            for (int t = 0; t < d; ++t) acc += q[t] * (double)bf2f(K[j * d + t]);
            s[j] = acc * scale;
            if (s[j] > mx) mx = s[j];
        }
        double l = 0.0;
        double *o = out + r * d;
        for (int t = 0; t < d; ++t) o[t] = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            if (!use[j]) continue;
            double p = exp(s[j] - mx);
            l += p;
            for (int t = 0; t < d; ++t) o[t] += p * (double)bf2f(V[j * d + t]);
        }
        for (int t = 0; t < d; ++t) o[t] /= l;
        free(s);
        free(use);
        free(q);
    }
}

/* Per key cluster c < nk: count and mean of the member rows (bf16 -> fp32),
 * members summed in ascending token order in fp32 and divided by the count,
 * as the Lloyd update does; empty clusters get count 0 and mean 0. */
void or_cluster_means(const uint16_t *X, int L, int d, const int32_t *labels, int nk, float *mean,
                      int32_t *count)
{
    for (int c = 0; c < nk; ++c) count[c] = 0;
    for (int64_t i = 0; i < (int64_t)nk * d; ++i) mean[i] = 0.0f;
    for (int64_t j = 0; j < L; ++j) {
        const int c = labels[j];
        if (c < 0 || c >= nk) continue;
        count[c] += 1;
        for (int t = 0; t < d; ++t) mean[(int64_t)c * d + t] = mean[(int64_t)c * d + t] + bf2f(X[j * d + t]);
    }
    for (int c = 0; c < nk; ++c)
        if (count[c] > 0)
            for (int t = 0; t < d; ++t) mean[(int64_t)c * d + t] = mean[(int64_t)c * d + t] / (float)count[c];
}

/* Centroid ("stripe-mean") compensation of the clusters a query cluster does
 * not select (ClusterAttention Sec. 1.2, Eq. (5)-(6)): for query row i of
 * query cluster qc, the keys of the selected clusters enter the softmax as in
 * or_attention_rows, and every other non-empty key cluster c < nk enters as
 * one pseudo-token with key kbar_c, value vbar_c and multiplicity |c|, i.e.
 * with weight |c| exp(scale q . kbar_c).  Dense units: every key, nothing to
 * compensate.  fp64. */
void or_attention_rows_comp(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int L, int d,
                            const int32_t *labels_q, const int32_t *labels_k, const int32_t *sel,
                            int32_t k, int dense, double scale, const int64_t *rows, int64_t nrows,
                            int nk, const int32_t *counts, const double *kbar, const double *vbar,
                            double *out)
{
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = rows[r];
        double *s = (double *)malloc((size_t)L * sizeof(double));
        double *sc = (double *)malloc((size_t)(nk > 0 ? nk : 1) * sizeof(double));
        char *chosen = (char *)calloc((size_t)(nk > 0 ? nk : 1), 1);
        double *q = (double *)malloc((size_t)d * sizeof(double));
        for (int t = 0; t < d; ++t) q[t] = (double)bf2f(Q[i * d + t]);
        if (dense) {
            for (int c = 0; c < nk; ++c) chosen[c] = 1;
        } else {
            const int32_t *my = sel + (int64_t)labels_q[i] * k;
            for (int a = 0; a < k; ++a)
                if (my[a] >= 0 && my[a] < nk) chosen[my[a]] = 1;
        }
        double mx = -INFINITY;
        for (int64_t j = 0; j < L; ++j) {
            const int c = labels_k[j];
            if (!(dense || (c >= 0 && c < nk && chosen[c]))) continue;
            double acc = 0.0;
            for (int t = 0; t < d; ++t) acc += q[t] * (double)bf2f(K[j * d + t]);
            s[j] = acc * scale;
            if (s[j] > mx) mx = s[j];
        }
        for (int c = 0; c < nk; ++c) {
            if (chosen[c] || counts[c] == 0) continue;
            double acc = 0.0;
            for (int t = 0; t < d; ++t) acc += q[t] * kbar[(int64_t)c * d + t];
            sc[c] = acc * scale + log((double)counts[c]);
            if (sc[c] > mx) mx = sc[c];
        }
        double l = 0.0;
        double *o = out + r * d;
        for (int t = 0; t < d; ++t) o[t] = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            const int c = labels_k[j];
            if (!(dense || (c >= 0 && c < nk && chosen[c]))) continue;
            double p = exp(s[j] - mx);
            l += p;
            for (int t = 0; t < d; ++t) o[t] += p * (double)bf2f(V[j * d + t]);
        }
        for (int c = 0; c < nk; ++c) {
            if (chosen[c] || counts[c] == 0) continue;
            double p = exp(sc[c] - mx);
            l += p;
            for (int t = 0; t < d; ++t) o[t] += p * vbar[(int64_t)c * d + t];
        }
        for (int t = 0; t < d; ++t) o[t] /= l;
        free(s);
        free(sc);
        free(chosen);
        free(q);
    }
}

/* Dense softmax weights of one query row over all L keys, fp64 (used by the
 * error-split self-check, ClusterAttention Sec. 1.2 Eq. (1)-(4)). */
void or_dense_weights(const uint16_t *q16, const uint16_t *K, int L, int d, double scale, double *w)
{
    double mx = -INFINITY;
    for (int64_t j = 0; j < L; ++j) {
        double acc = 0.0;
        for (int t = 0; t < d; ++t) acc += (double)bf2f(q16[t]) * (double)bf2f(K[j * d + t]);
        w[j] = acc * scale;
        if (w[j] > mx) mx = w[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < L; ++j) {
        w[j] = exp(w[j] - mx);
        l += w[j];
    }
    for (int64_t j = 0; j < L; ++j) w[j] /= l;
}
