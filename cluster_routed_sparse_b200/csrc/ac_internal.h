// ac_internal.h -- context layout and kernel launchers of libac (host side).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <string>

#include "ac.h"

typedef __nv_bfloat16 bf16;

struct ac_ctx {
    ac_config cfg;
    int B, H, L, d, BH, Cq, Ccap;
    int device;
    float scale;

    // ---- query clustering (Algorithm 3 line 3)
    float *inv_q;      // [BH, L]
    int *labels_q;     // [BH, L]
    float *cent_q;     // [BH, Cq, d]
    int *counts_q;     // [BH, Cq]
    int *perm_q;       // [BH, L]
    int *offs_q;       // [BH, Cq+1]

    // ---- key clustering (Algorithm 1)
    int *labels_k;     // [BH, L]
    float *dmin_k;     // [BH, L]
    float *cent_k;     // [BH, Ccap, d]
    int *n_k;          // [BH]
    uint8_t *dense;    // [BH]
    int *stages;       // [BH]
    int *fallback_at;  // [BH] cluster count at the head of the last stage (see AC_T_FALLBACK_AT)
    int *removed_stage;  // [BH, L]
    float *tau;        // [1]
    unsigned long long *tau_acc;  // [1] fixed-point sum of stage-0 distances
    int *counts_k;     // [BH, Ccap]
    int *perm_k;       // [BH, L]
    int *offs_k;       // [BH, Ccap+1]
    bf16 *kmax, *kmin; // [BH, Ccap, d]
    float *sse;        // [BH, Ccap]
    float *mse, *comp; // [BH]

    // ---- multi-stage scratch
    int *u_idx;        // [BH, L]  unabsorbed keys, ascending
    int *u_idx2;       // [BH, L]
    int *u_cnt;        // [BH]
    int *st_m;         // [BH]     clusters of the current stage (0: idle head)
    int *st_labels;    // [BH, L]
    float *st_dist;    // [BH, L]
    int *st_perm;      // [BH, L]
    int *st_offs;      // [BH, m0+1]
    int *st_counts;    // [BH, m0]
    uint32_t *radix;   // [256 + 4] percentile selection scratch
    int *sort_scratch; // [BH, 129, max(Ccap, Cq)] counting-sort chunk histograms and label totals

    // ---- selection (Algorithm 3 line 9)
    float *score;      // [BH, Cq, Ccap]
    float *kabs;       // [BH, Ccap]      max_d max(|Kmax_d|, |Kmin_d|) per key cluster
    CUtensorMap tm_kmax, tm_kmin;  // Kmax / Kmin rows in 64-row boxes (tensor-core Eq. (1))
    int *sel;          // [BH, Cq, Ccap]
    int *ksel;         // [BH]
    int2 *ranges;      // [BH, Cq, Ccap]  (start row in cluster order, count)
    int *nboxes;       // [BH*Cq]         8-row key boxes per query cluster
    int *rbox;         // [BH*Cq, Ccap+1] first box of each selected range (exclusive prefix)
    int *tile_prefix;  // [BH*Cq+1]       attention items (pairs of 128-query tiles), exclusive prefix
    // tail merging (cfg.tail_merge != 0): the attention's query layout by group
    int *perm_qm;      // [BH, L]   token of each row of Qp
    int *offs_qm;      // [BH, Cq+1] first row of each group (owner cluster id)
    int *counts_qm;    // [BH, Cq]  rows of each group (0: merged into another)
    int *tm_scratch;   // [4, BH, Cq] owner, position in group, rows kept, base of handed rows
    // centroid compensation (cfg.compensate): member means of every key cluster,
    // written as bf16 rows of a centroid block of Kp / Vp (group cgroup of each
    // unit), one key range over that block per query cluster (crange), and the
    // block's per-column addends ln|c| / scale, -inf for the selected clusters
    float *kbar, *vbar;  // [BH, Ccap, d]
    float *cbias;        // [BH, Cq, Ccap]
    int *crange;         // [BH*Cq]  index of the centroid range, -1: none
    int cgroup;          // first 8-row group of the centroid block within a unit of Kp / Vp

    // ---- tensor-core assignment (centres split into bf16 + remainder)
    int Cpad_q, CH_q, Cpad_k, CH_k;  // padded centre rows per unit, centres per chunk
    bf16 *chi_q, *chi_k;  // [2, BH, Cpad_q, d] c_hi, c_lo of the query centres; [BH, Cpad_k, d] c_hi of the key centres
    float *cn;         // [BH, max Cpad] |c_hi|^2
    unsigned int *hstat;  // [BH, 2]
    float *rowsq_k;    // [BH, L] |k|^2
    int4 *cand;        // [BH * L] candidates of uncertain rows
    int *amb_list;     // [BH * L]
    int *amb_count;    // [1]
    unsigned long long *asg_stats;  // [2] uncertain rows, rows rescored against every centre
    CUtensorMap tm_chi_q, tm_chi_k;
    bf16 *cnp_k;       // [BH, Cpad_k, 16] |c'|^2 of the key centres as three bf16 parts
    CUtensorMap tm_cnp_k;
    CUtensorMap tm_xq, tm_xk;  // caller's Q / K of the current call
    CUtensorMap tm_xu;         // gathered keys of a stage t >= 1 (rows of Qp, which is free then)
    float *rowsq_u;            // [BH, L] |k|^2 of the gathered keys, by position in U
    float *cent_st;            // [BH, m0, d] the stage's centres, copied out of cent_k for the GEMM
    int num_sms;
    bool fast_assign;
    bool exact_scores;  // Eq. (1) on CUDA cores instead of the tensor cores
    float quest_bound_scale;  // >= 1: the tensor-core Eq. (1) path rescores a wider band
    long long n_fast, n_exact, n_fast_rows;

    // ---- attention
    bf16 *Qp;          // [BH, L, d] queries in cluster order
    bf16 *Kp, *Vp;     // [BH, Lpad, d] keys / values in cluster order, every key
                       // cluster starting on an 8-row group (padding rows zero)
    int Lpad;          // rows per unit of Kp / Vp: L rounded up to 8, plus 8 per cluster
    int *pgoff;        // [BH, Ccap] first 8-row group of each key cluster in Kp / Vp
    int *nrange;       // [BH*Cq] key ranges the attention walks (k, or all clusters when dense)
    unsigned long long *counters;  // [8] kept pairs, computed pairs, items, -, first wait failure
    CUtensorMap tm_q;
    CUtensorMap tm_kg[4], tm_vg[4];  // K / V boxes of 1, 2, 4, 8 row groups

    // ---- host-buffer forward
    uint16_t *hbufQ, *hbufK, *hbufV, *hbufO;  // device staging of the host entry point
    // asynchronous host entry point: two staging sets (Q, K, V, O each), an
    // input-copy and an output-copy stream, and per set the events "inputs
    // landed", "layer done" and "output copied"
    uint16_t *abuf[2][4];
    cudaStream_t s_in, s_out;
    cudaEvent_t ev_in[2], ev_comp[2], ev_out[2];
    cudaEvent_t ev_inq[2], ev_ink[2];  // Q landed, K landed (ev_in: V, the last)
    long long async_calls;

    uint32_t *err;      // device error word
    int *h_u_cnt;       // pinned host mirrors
    int *h_st_m;
    int *h_n_k;
    uint8_t *h_dense;
    uint32_t *h_err;
    uint64_t *h_xchg;   // [256] u64 + [256] u32: the tau exchange's partial sums
    ac_sum_u64_fn xchg = nullptr;  // sums partial results over the contexts of one layer
    void *xchg_user = nullptr;

    bool have_q, have_k, have_state;
    bool timing;        // record events around the attention kernel
    std::string msg;
    cudaEvent_t ev[8];
};

// ---------------------------------------------------------------- launchers
// All launchers enqueue on `s` and return the launch status.
namespace ac {

// Kernels launched by this library in this process.
extern std::atomic<long long> g_launches;
#define AC_NOTE_LAUNCH() ::ac::g_launches.fetch_add(1, std::memory_order_relaxed)

// Message returned by ac_last_error_string(NULL) (per thread).
void set_static_error(const char *msg);

cudaError_t launch_qnorm(const bf16 *Q, float *inv, int64_t rows, int d, uint32_t *err, cudaStream_t s);

// Exact assignment: for every row of every unit h (rows given by an index
// list or 0..n-1), label = argmin over the unit's centres of the fp32
// squared distance summed in dimension order; ties to the lowest index.
struct AssignArgs {
    const bf16 *X;        // [BH, L, d]
    const float *inv;     // [BH, L] or null (then rows are not normalised)
    int64_t L;
    const int *rows;      // [BH, L] row indices or null
    const int *nrows;     // [BH] or null (then nrows_const)
    int nrows_const;
    const float *C;       // [BH, cstride] centres
    int64_t cstride;      // floats per unit
    const int *coff;      // [BH] first centre of the unit (in centres) or null
    const int *ncent;     // [BH] or null (then ncent_const)
    int ncent_const;
    int *labels;          // [BH, L]
    float *dmin;          // [BH, L] or null
    int BH, d;
};
cudaError_t launch_assign_exact(const AssignArgs &a, cudaStream_t s);

// The same labels from the tensor cores (see assign_mma.cu): rows 0..n-1 of
// every unit, centres 0..m-1 of the unit at C + h * cstride.
struct FastAssignArgs {
    const CUtensorMap *tm_x;   // rows [BH * L, d], box {64, 128}
    const CUtensorMap *tm_c;   // Chi rows [BH * Cpad (x2 with two terms), d], box {64, CH}
    const CUtensorMap *tm_cn;  // cnp [BH * Cpad, 16] bf16, box {8, CH}, no swizzle (keys only)
    const bf16 *X;
    const float *inv;          // [BH, L] or null
    const float *rowsq;        // [BH, L] |x|^2 when inv is null
    int64_t L;
    const int *nrows; int nrows_const;
    const float *C; int64_t cstride;
    const int *ncent; int ncent_const;
    int Cpad, CH;              // CH <= 128, <= 96 with two terms
    bool two_term;             // centres as bf16 c_hi + c_lo (else c_hi alone)
    bf16 *Chi; bf16 *cnp; float *cn; unsigned int *hstat;
    int *labels;
    float *dmin;               // or null
    int4 *cand; int *amb_list; int *amb_count;
    unsigned long long *stats;
    uint32_t *err;
    int BH, d, num_sms;
};
cudaError_t launch_assign_fast(const FastAssignArgs &a, cudaStream_t s);
cudaError_t launch_row_sqnorm(const bf16 *X, int64_t rows, int d, float *out, cudaStream_t s);

// Stable counting sort of labels per unit: perm[h, pos] = row position (or
// rows[pos]'s index when rows given, see below), offs[h, 0..m], counts[h, 0..m).
struct SortArgs {
    const int *labels;    // [BH, L]
    int64_t L;
    const int *nrows;     // [BH] or null
    int nrows_const;
    const int *nlab;      // [BH] or null
    int nlab_const;
    int max_lab;          // upper bound of nlab over units
    int *perm;            // [BH, L]
    int *offs;            // [BH, offs_stride]
    int offs_stride;
    int *counts;          // [BH, counts_stride] or null
    int counts_stride;
    int BH;
    int *scratch;         // [BH, 128, max_lab] per-chunk histograms / slots, then [BH, max_lab] label totals
};
cudaError_t launch_counting_sort(const SortArgs &a, cudaStream_t s);

// Centre update: C[h, coff+c] = mean of the members of cluster c, summed in
// ascending order; empty clusters keep their centre.
struct UpdateArgs {
    const bf16 *X; const float *inv; int64_t L;
    const int *rows;      // [BH, L] or null
    const int *perm; const int *offs; int offs_stride;
    float *C; int64_t cstride; const int *coff;
    const int *ncent; int ncent_const;
    int BH, d, max_cent;
    uint32_t *err = nullptr;  // bounded-wait failures are recorded here
};
cudaError_t launch_update(const UpdateArgs &a, cudaStream_t s);

// Seeded initial centres: C[h, coff + j] = X[rows[h, pick_j]] (normalised
// when inv is given), j < m[h], pick_j from stratum j of n[h] members.
struct SeedArgs {
    const bf16 *X; const float *inv; int64_t L;
    const int *rows; const int *nrows; int nrows_const;
    float *C; int64_t cstride; const int *coff;
    const int *m; int m_const; int max_m;
    uint64_t seed; int tag; int BH, d;
    int unit0 = 0;  // unit index of the first unit (a head subset of a larger layer)
};
cudaError_t launch_seed(const SeedArgs &a, cudaStream_t s);

// Multi-stage helpers.
cudaError_t launch_iota_rows(int *u_idx, int *u_cnt, int BH, int L, cudaStream_t s);
cudaError_t launch_stage_dist(const float *dmin, float *dist, const int *u_cnt, const int *st_m,
                              int64_t L, int BH, unsigned long long *tau_acc, cudaStream_t s);
cudaError_t launch_tau_mean(const unsigned long long *tau_acc, const int *u_cnt0_total_unused,
                            int64_t n_total, float factor, float *tau, cudaStream_t s);
cudaError_t launch_radix_hist(const float *dist, const int *st_m, int64_t L, int BH, uint32_t *radix, int shift,
                              cudaStream_t s);
cudaError_t launch_tau_percentile(const float *dist, const int *st_m, int64_t L, int BH,
                                  int64_t n_total, int permille, uint32_t *radix, float *tau,
                                  cudaStream_t s);
cudaError_t launch_remove(const float *dist, const float *tau, int *u_idx, int *u_idx2, int *u_cnt,
                          const int *st_m, int *removed_stage, int stage, int64_t L, int BH,
                          cudaStream_t s);

// Also writes dmin[h, t] = exact squared distance of key t to its centre.
struct StatsArgs {
    const bf16 *K; int64_t L; const int *perm; const int *offs; int offs_stride;
    float *dmin; const int *n_k; int Ccap; int d; int BH;
    int *counts; bf16 *kmax; bf16 *kmin; float *sse; float *mse; float *comp;
    const float *C; int64_t cstride;  // key centres
    uint32_t *err;
    float *dsorted;                   // [BH, L] scratch: the distances in member order
};
cudaError_t launch_key_stats(const StatsArgs &a, cudaStream_t s);

cudaError_t launch_permute_rows(const bf16 *X, const int *perm, bf16 *Xp, int64_t L, int d, int BH,
                                cudaStream_t s);
// Kp / Vp row 8 pgoff[h, c] + i = K / V row of the i-th key of cluster c.
cudaError_t launch_permute_kv_padded(const bf16 *K, const bf16 *V, const int *perm, const int *labels,
                                     const int *offs, int offs_stride, const int *pgoff, int Ccap, bf16 *Kp,
                                     bf16 *Vp, int64_t L, int64_t Lpad, int d, int BH, cudaStream_t s);

struct SelectArgs {
    const float *cent_q; const bf16 *kmax; const bf16 *kmin; const int *counts_k;
    const int *n_k; const uint8_t *dense; const int *offs_k; const int *counts_q;
    int Cq, Ccap, d, BH, L, topk;
    float *score; int *sel; int *ksel; int2 *ranges; int *nboxes; int *tile_prefix;
    int *rbox; int *pgoff; int *nrange;
    int score_mode = 0;            // 0: Eq. (1) bound; 1: mean-based (q . centre of the key cluster)
    const float *cent_k = nullptr;  // [BH, Ccap, d] key centres (score_mode 1)
    // tensor-core path of Eq. (1) (quest_mma.cu): Kmax / Kmin rows [BH * Ccap, d]
    // in 64-row boxes, the per-cluster column bounds, the error word
    const CUtensorMap *tm_kmax = nullptr, *tm_kmin = nullptr;
    float *kabs = nullptr;         // [BH, Ccap]
    uint32_t *err = nullptr;
    bool exact_cuda_cores = false;  // force the CUDA-core kernels (k_quest_scores + k_score_select)
    // centroid compensation: per-column addends and the extra key range (null: off)
    float *cbias = nullptr; int *crange = nullptr; int cgroup = 0; float scale = 1.f;
    float bound_scale = 1.f;        // widens the tensor-core path's error bound (tests of the rescoring)
};
cudaError_t launch_score_select(const SelectArgs &a, cudaStream_t s);
bool quest_mma_supported(const SelectArgs &a);
cudaError_t launch_quest_select_mma(const SelectArgs &a, cudaStream_t s);

// Tail merging of the query tiles after the selection (see ac_config.tail_merge):
// regroups the rows of Qp (perm_qm, offs_qm, counts_qm), rewrites the key
// ranges of the clusters that take another's tail, and the attention items.
struct TailMergeArgs {
    const int *sel; const int *ksel; const uint8_t *dense;
    const int *labels_q; const int *perm_q; const int *offs_q; const int *counts_q;
    const int *counts_k; const int *pgoff;
    int2 *ranges; int *rbox; int *nrange; int *nboxes;
    int *perm_qm; int *offs_qm; int *counts_qm; int *scratch; int *tile_prefix;
    int Cq, Ccap, BH, mode;
    int64_t L;
};
cudaError_t launch_tail_merge(const TailMergeArgs &a, cudaStream_t s);

struct AttnArgs {
    const CUtensorMap *tm_q, *tm_kg, *tm_vg;  // tm_kg / tm_vg: [4] box sizes
    bf16 *O; const int *perm_q; const int *offs_q; const int *counts_q;
    const int *tile_prefix; const int2 *ranges; const int *nboxes; const int *nrange; const int *rbox;
    int L, Lpad, Cq, Ccap, BH, d;
    float scale_log2;
    uint32_t *err; unsigned long long *counters;
    const int *crange = nullptr; const float *cbias = nullptr;  // centroid compensation (null: off)
};
cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t s);
// bf16 rows of the centroid block: Kp / Vp row 8 cgroup + c of unit h = kbar / vbar [h, c], c < n_k[h]
cudaError_t launch_comp_rows(const float *kbar, const float *vbar, const int *n_k, int Ccap, int d, int BH,
                             int64_t Lpad, int cgroup, bf16 *Kp, bf16 *Vp, cudaStream_t s);
int attn_max_tiles(int L, int Cq, int BH);

}  // namespace ac
