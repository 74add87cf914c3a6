// ac_api.cu -- the C ABI of libac: context, workspace, and the host control
// flow of the cluster-routed sparse layer (AdaCluster, arXiv 2604.18348,
// Algorithm 3, with Algorithm 1 for the keys).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <functional>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "ac_device.cuh"
#include "ac_internal.h"

using namespace ac;

std::atomic<long long> ac::g_launches{0};

namespace {

thread_local std::string g_static_msg;

ac_status fail(ac_ctx *c, ac_status st, const char *what) {
    if (c) c->msg = what;
    return st;
}

ac_status cuda_fail(ac_ctx *c, cudaError_t e, const char *what) {
    if (c) {
        char buf[512];
        snprintf(buf, sizeof(buf), "%s: %s", what, cudaGetErrorString(e));
        c->msg = buf;
    }
    return AC_ERR_CUDA;
}

#define CK(call, what)                                   \
    do {                                                 \
        cudaError_t e_ = (call);                         \
        if (e_ != cudaSuccess) return cuda_fail(c, e_, what); \
    } while (0)

// Cluster count m_t of stage t (Algorithm 1 line 11, "choose a moderate
// cluster number"): rule 0 makes the stage-0 choice every stage, min(m0, |U|);
// rule 1 keeps the mean cluster size at L/m0, ceil(m0 |U| / L).
int stage_clusters(int m0, int64_t nU, int64_t L, int t, int rule) {
    if (t == 0 || rule == 0) return (int)std::min<int64_t>(m0, nU);
    int64_t m = (m0 * nU + L - 1) / L;
    m = std::max<int64_t>(1, std::min<int64_t>(m, nU));
    return (int)m;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

ac_status make_tmap(ac_ctx *c, CUtensorMap *tm, void *base, int64_t rows, int d, int box_rows) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(c, AC_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(c, AC_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    return AC_OK;
}

// Rows of 16 bf16, boxes of 8 columns x box_rows rows, no swizzle: in shared
// memory a box is box_rows x 16 bytes, i.e. 8-row x 16-byte core matrices
// one after the other.
ac_status make_tmap_plain16(ac_ctx *c, CUtensorMap *tm, void *base, int64_t rows, int box_rows) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(c, AC_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    cuuint64_t dims[2] = {16, (cuuint64_t)rows};
    cuuint64_t strides[1] = {32};
    cuuint32_t box[2] = {8, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(c, AC_ERR_CUDA, "cuTensorMapEncodeTiled (norm parts) failed");
    return AC_OK;
}

// K and V boxes of G 8-row groups x all d columns in one copy, laid out in
// shared memory as [group][column half][8 rows][64 columns] (dims: column,
// row in group, half, group; strides d*2, 128 and 8*d*2 bytes), 128-byte
// swizzle.  The rows must be group-aligned, as the padded Kp / Vp are.
ac_status make_tmap_kv(ac_ctx *c, CUtensorMap *tm, void *base, int64_t groups, int d, int G) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(c, AC_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found");
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    const int halves = d / 64;
    cuuint64_t dims[4] = {64, 8, (cuuint64_t)halves, (cuuint64_t)groups};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, 128, (cuuint64_t)d * 16};
    cuuint32_t box[4] = {64, 8, (cuuint32_t)halves, (cuuint32_t)G};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(c, AC_ERR_CUDA, "cuTensorMapEncodeTiled (K/V group boxes) failed");
    return AC_OK;
}

template <class T>
cudaError_t dalloc(T **p, size_t n) {
    return cudaMalloc(reinterpret_cast<void **>(p), std::max<size_t>(n, 1) * sizeof(T));
}

// Read back the device error word, clear it, and turn it into a status.
ac_status check_dev_err(ac_ctx *c, cudaStream_t s) {
    CK(cudaMemcpyAsync(c->h_err, c->err, sizeof(uint32_t), cudaMemcpyDeviceToHost, s), "error word");
    CK(cudaStreamSynchronize(s), "stream sync");
    uint32_t e = *c->h_err;
    if (e) {
        CK(cudaMemsetAsync(c->err, 0, sizeof(uint32_t), s), "error word reset");
        if (e & DEV_ERR_NONFINITE) return fail(c, AC_ERR_NONFINITE, "non-finite value in an input");
        if (e & DEV_ERR_TIMEOUT) return fail(c, AC_ERR_TIMEOUT, "a bounded in-kernel wait expired");
        return fail(c, AC_ERR_CUDA, "kernel bounds check failed");
    }
    return AC_OK;
}

// ---------------------------------------------------------------- k-means pieces
// T Lloyd iterations (assign, sort, update) then a final assignment + sort.
struct Lloyd {
    AssignArgs as;
    SortArgs so;
    UpdateArgs up;
    bool fast = false;  // assignment on the tensor cores (fa) instead of the exact kernel (as)
    FastAssignArgs fa;
    bool stage_copy = false;  // copy the stage centres out of cent_k before each tensor-core pass
    long long rows = -1;      // rows one pass assigns (for the counters), when not every row of every unit
};

// Stage centres of unit h (cent_k rows n_k[h] .. n_k[h] + m[h] - 1) into the
// compact [BH, m0, d] buffer the tensor-core assignment reads.
__global__ void k_stage_centres(const float *__restrict__ C, int64_t cstride, const int *__restrict__ n_k,
                                const int *__restrict__ m, int m0, int d, float *__restrict__ out) {
    const int c = blockIdx.x, h = blockIdx.y;
    if (c >= m[h]) return;
    const float *src = C + (int64_t)h * cstride + (int64_t)(n_k[h] + c) * d;
    float *dst = out + ((int64_t)h * m0 + c) * d;
    for (int k = threadIdx.x; k < d; k += blockDim.x) dst[k] = src[k];
}

// Xg[h, pos] = X[h, idx[h, pos]] for pos < cnt[h], and sq[h, pos] = |Xg[h, pos]|^2
// (fp32; it only enters the assignment's error bound).  d / 8 lanes per row.
__global__ void k_gather_rows_sq(const bf16 *__restrict__ X, const int *__restrict__ idx, const int *__restrict__ cnt,
                                 bf16 *__restrict__ Xg, float *__restrict__ sq, int64_t L, int d) {
    const int h = blockIdx.y;
    const int lpr = d / 8;  // lanes per row (8 or 16), a power of two dividing 32
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t pos = g / lpr;
    const int part = (int)(g % lpr);
    const bool v = pos < cnt[h];
    float ss = 0.f;
    if (v) {
        const int64_t src = (int64_t)h * L + idx[(int64_t)h * L + pos];
        const uint4 w = reinterpret_cast<const uint4 *>(X + src * d)[part];
        reinterpret_cast<uint4 *>(Xg + ((int64_t)h * L + pos) * d)[part] = w;
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        for (int t = 0; t < 4; ++t) {
            const float a = __uint_as_float(ws[t] << 16), b = __uint_as_float(ws[t] & 0xFFFF0000u);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
        }
    }
    for (int o = lpr / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (v && part == 0) sq[(int64_t)h * L + pos] = ss;
}

// One assignment pass; dmin (where the caller asked for it) only when wanted.
cudaError_t assign_pass(ac_ctx *c, const Lloyd &k, bool want_dmin, cudaStream_t s) {
    if (k.fast) {
        if (k.stage_copy) {
            k_stage_centres<<<dim3(c->cfg.m0, c->BH), 128, 0, s>>>(c->cent_k, (int64_t)c->Ccap * c->d, c->n_k,
                                                                   c->st_m, c->cfg.m0, c->d, c->cent_st);
            AC_NOTE_LAUNCH();
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        FastAssignArgs a = k.fa;
        if (!want_dmin) a.dmin = nullptr;
        ++c->n_fast;
        c->n_fast_rows += k.rows >= 0 ? k.rows : (long long)a.BH * a.L;
        return launch_assign_fast(a, s);
    }
    ++c->n_exact;
    return launch_assign_exact(k.as, s);
}

cudaError_t run_lloyd(ac_ctx *c, Lloyd &k, int T, bool final_sort, cudaStream_t s, bool final_dmin = true) {
    cudaError_t e;
    k.up.err = c->err;
    for (int t = 0; t < T; ++t) {
        if ((e = assign_pass(c, k, false, s)) != cudaSuccess) return e;
        if ((e = launch_counting_sort(k.so, s)) != cudaSuccess) return e;
        if ((e = launch_update(k.up, s)) != cudaSuccess) return e;
    }
    if ((e = assign_pass(c, k, final_dmin, s)) != cudaSuccess) return e;
    if (final_sort && (e = launch_counting_sort(k.so, s)) != cudaSuccess) return e;
    return cudaSuccess;
}

// Tensor-core assignment of all rows 0..L-1 of every unit against the unit's
// centres 0..m-1 at C + h * cstride (see assign_mma.cu).  Returns false (exact
// kernel instead) when disabled or when the rows are not 16-byte aligned.
bool make_fast(ac_ctx *c, Lloyd &k, const bf16 *X, bool queries, const float *C, int64_t cstride,
               const int *ncent, int ncent_const, int *labels, float *dmin) {
    if (!c->fast_assign || (reinterpret_cast<uintptr_t>(X) & 15u) != 0) return false;
    CUtensorMap *tmx = queries ? &c->tm_xq : (X == c->Qp ? &c->tm_xu : &c->tm_xk);
    if (make_tmap(c, tmx, const_cast<bf16 *>(X), (int64_t)c->BH * c->L, c->d, 128) != AC_OK) return false;
    FastAssignArgs &a = k.fa;
    a.tm_x = tmx;
    a.tm_c = queries ? &c->tm_chi_q : &c->tm_chi_k;
    a.tm_cn = queries ? nullptr : &c->tm_cnp_k;
    a.cnp = queries ? nullptr : c->cnp_k;
    a.X = X;
    a.inv = queries ? c->inv_q : nullptr;
    a.rowsq = queries ? nullptr : c->rowsq_k;
    a.L = c->L;
    a.nrows = nullptr;
    a.nrows_const = c->L;
    a.C = C;
    a.cstride = cstride;
    a.ncent = ncent;
    a.ncent_const = ncent_const;
    a.Cpad = queries ? c->Cpad_q : c->Cpad_k;
    a.CH = queries ? c->CH_q : c->CH_k;
    a.Chi = queries ? c->chi_q : c->chi_k;
    // Normalised queries sit in tight angular clusters (distances ~1e-2 of
    // |x|^2): c_hi alone would leave most rows to the exact rescoring.
    a.two_term = queries;
    a.cn = c->cn;
    a.hstat = c->hstat;
    a.labels = labels;
    a.dmin = dmin;
    a.cand = c->cand;
    a.amb_list = c->amb_list;
    a.amb_count = c->amb_count;
    a.stats = c->asg_stats;
    a.err = c->err;
    a.BH = c->BH;
    a.d = c->d;
    a.num_sms = c->num_sms;
    k.fast = true;
    return true;
}

// Algorithm 3 line 3 on the context's buffers.
ac_status cluster_q_impl(ac_ctx *c, const bf16 *Q, const float *init, int iters, cudaStream_t s) {
    const int64_t L = c->L;
    CK(launch_qnorm(Q, c->inv_q, (int64_t)c->BH * L, c->d, c->err, s), "qnorm");
    if (init) {
        if (init != c->cent_q)
            CK(cudaMemcpyAsync(c->cent_q, init, sizeof(float) * c->BH * c->Cq * c->d, cudaMemcpyDeviceToDevice, s),
               "init copy");
    } else {
        SeedArgs sa{Q, c->inv_q, L, nullptr, nullptr, c->L, c->cent_q, (int64_t)c->Cq * c->d, nullptr,
                    nullptr, c->Cq, c->Cq, c->cfg.seed, 0, c->BH, c->d};
        sa.unit0 = c->cfg.unit0;
        CK(launch_seed(sa, s), "seed q");
    }
    Lloyd k;
    k.as = AssignArgs{Q, c->inv_q, L, nullptr, nullptr, c->L, c->cent_q, (int64_t)c->Cq * c->d, nullptr,
                      nullptr, c->Cq, c->labels_q, nullptr, c->BH, c->d};
    k.so = SortArgs{c->labels_q, L, nullptr, c->L, nullptr, c->Cq, c->Cq, c->perm_q, c->offs_q, c->Cq + 1,
                    c->counts_q, c->Cq, c->BH, c->sort_scratch};
    k.up = UpdateArgs{Q, c->inv_q, L, nullptr, c->perm_q, c->offs_q, c->Cq + 1, c->cent_q,
                      (int64_t)c->Cq * c->d, nullptr, nullptr, c->Cq, c->BH, c->d, c->Cq};
    make_fast(c, k, Q, true, c->cent_q, (int64_t)c->Cq * c->d, nullptr, c->Cq, c->labels_q, nullptr);
    CK(run_lloyd(c, k, iters, true, s), "q lloyd");
    c->have_q = true;
    return AC_OK;
}

// The pooled tau when the heads of one layer are split over several contexts
// (ranks): each context reduces its own stage-0 distances and the caller's
// exchange function sums the partial results over the contexts, so tau is the
// one a single context over all heads computes, bit for bit (the fixed-point
// sum and the radix-select histograms are order-independent integers).
//  mean rule:       {sum floor(d_i 2^24), n}, then tau on the host as k_tau_mean forms it;
//  percentile rule: {n}, then per 8-bit digit the 256-bin histogram of the
//                   distances that match the digits chosen so far.
ac_status exchange_tau(ac_ctx *c, cudaStream_t s) {
    const int BH = c->BH, L = c->L;
    uint64_t *hx = c->h_xchg;
    float tau = 0.f;
    if (c->cfg.tau_mode == AC_TAU_MEAN_FACTOR) {
        CK(cudaMemcpyAsync(hx, c->tau_acc, sizeof(uint64_t), cudaMemcpyDeviceToHost, s), "tau partial");
        CK(cudaStreamSynchronize(s), "tau partial");
        hx[1] = (uint64_t)BH * (uint64_t)L;
        if (c->xchg(c->xchg_user, hx, 2) != 0) return fail(c, AC_ERR_STATE, "tau exchange function failed");
        ac_status st = ac_tau_mean_from_sums(c->cfg.tau_value, hx[0], hx[1], &tau);
        if (st != AC_OK) return fail(c, st, "tau exchange: no distances");
    } else {
        hx[0] = (uint64_t)BH * (uint64_t)L;
        if (c->xchg(c->xchg_user, hx, 1) != 0) return fail(c, AC_ERR_STATE, "tau exchange function failed");
        const uint64_t n_total = hx[0];
        if (n_total == 0 || n_total > 0xFFFFFFFFull) return fail(c, AC_ERR_INVALID_ARG, "tau exchange: bad key count");
        int64_t idx = ((int64_t)c->cfg.tau_value * (int64_t)n_total + 999) / 1000 - 1;
        idx = std::max<int64_t>(0, std::min<int64_t>(idx, (int64_t)n_total - 1));
        uint32_t state[3] = {0u, 0u, (uint32_t)idx};  // prefix, mask, rank within the prefix
        uint32_t *hh = reinterpret_cast<uint32_t *>(hx + 256);
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            uint32_t init[259];
            for (int i = 0; i < 256; ++i) init[i] = 0u;
            init[256] = state[0];
            init[257] = state[1];
            init[258] = state[2];
            CK(cudaMemcpyAsync(c->radix, init, sizeof(init), cudaMemcpyHostToDevice, s), "radix state");
            CK(launch_radix_hist(c->st_dist, c->st_m, L, BH, c->radix, shift, s), "radix histogram");
            CK(cudaMemcpyAsync(hh, c->radix, 256 * sizeof(uint32_t), cudaMemcpyDeviceToHost, s), "histogram");
            CK(cudaStreamSynchronize(s), "histogram");
            for (int i = 0; i < 256; ++i) hx[i] = hh[i];
            if (c->xchg(c->xchg_user, hx, 256) != 0) return fail(c, AC_ERR_STATE, "tau exchange function failed");
            ac_status st = ac_tau_radix_pick(hx, shift, state);
            if (st != AC_OK) return fail(c, st, "tau exchange: inconsistent histograms");
        }
        std::memcpy(&tau, &state[0], sizeof(float));
    }
    CK(cudaMemcpyAsync(c->tau, &tau, sizeof(float), cudaMemcpyHostToDevice, s), "tau");
    CK(cudaStreamSynchronize(s), "tau");  // `init` and the pinned buffer are reused
    return AC_OK;
}

// Algorithm 1, step 0 (all units batched; one readback of |U| per stage).
// The loop state lives in host vectors; the pinned staging buffers are only
// rewritten after a stream synchronisation, so no pending copy reads them.
ac_status cluster_k_step0(ac_ctx *c, const bf16 *K, cudaStream_t s) {
    const int BH = c->BH, L = c->L, d = c->d, m0 = c->cfg.m0;
    const int64_t cstride = (int64_t)c->Ccap * d;
    if (c->fast_assign) CK(launch_row_sqnorm(K, (int64_t)BH * L, d, c->rowsq_k, s), "row norms");
    CK(launch_iota_rows(c->u_idx, c->u_cnt, BH, L, s), "iota");
    CK(cudaMemsetAsync(c->removed_stage, 0xFF, sizeof(int) * BH * (size_t)L, s), "removed init");
    CK(cudaMemsetAsync(c->tau_acc, 0, sizeof(unsigned long long), s), "tau acc");
    std::vector<int> done(BH, 0), stages(BH, 0), nk(BH, 0), m(BH, 0), ucnt(BH, L), m_last(BH, 0);
    std::vector<uint8_t> dense(BH, 0);
    for (int t = 0;; ++t) {
        if (t > 0) {
            CK(cudaMemcpyAsync(c->h_u_cnt, c->u_cnt, sizeof(int) * BH, cudaMemcpyDeviceToHost, s), "u_cnt");
            CK(cudaStreamSynchronize(s), "stage sync");
            for (int h = 0; h < BH; ++h) {
                ucnt[h] = c->h_u_cnt[h];
                nk[h] += m[h];  // line 19 of the previous stage
            }
        }
        bool any = false;
        int max_m = 0;
        for (int h = 0; h < BH; ++h) {
            m[h] = 0;
            if (done[h]) continue;
            if (ucnt[h] == 0) {            // line 6: U is empty
                done[h] = 1;
                stages[h] = t;
                continue;
            }
            if (nk[h] >= c->cfg.n_max) {  // lines 7-9
                dense[h] = 1;
                done[h] = 1;
                stages[h] = t;
                continue;
            }
            m[h] = stage_clusters(m0, ucnt[h], L, t, c->cfg.stage_rule);  // line 11
            m_last[h] = m[h];
            max_m = std::max(max_m, m[h]);
            any = true;
        }
        if (!any) break;
        for (int h = 0; h < BH; ++h) {
            c->h_st_m[h] = m[h];
            c->h_n_k[h] = nk[h];
        }
        CK(cudaMemcpyAsync(c->st_m, c->h_st_m, sizeof(int) * BH, cudaMemcpyHostToDevice, s), "st_m");
        CK(cudaMemcpyAsync(c->n_k, c->h_n_k, sizeof(int) * BH, cudaMemcpyHostToDevice, s), "n_k");
        // line 12: KMeans(U, m_t), stage centres appended after the n_k existing ones
        SeedArgs sa{K, nullptr, L, c->u_idx, c->u_cnt, 0, c->cent_k, cstride, c->n_k, c->st_m, 0, max_m,
                    c->cfg.seed, 1 + t, BH, d};
        sa.unit0 = c->cfg.unit0;
        CK(launch_seed(sa, s), "seed k");
        Lloyd k;
        k.as = AssignArgs{K, nullptr, L, c->u_idx, c->u_cnt, 0, c->cent_k, cstride, c->n_k, c->st_m, 0,
                          c->st_labels, c->dmin_k, BH, d};
        k.so = SortArgs{c->st_labels, L, c->u_cnt, 0, c->st_m, 0, max_m, c->st_perm, c->st_offs, m0 + 1, nullptr,
                        0, BH, c->sort_scratch};
        k.up = UpdateArgs{K, nullptr, L, c->u_idx, c->st_perm, c->st_offs, m0 + 1, c->cent_k, cstride, c->n_k,
                          c->st_m, 0, BH, d, max_m};
        // stage 0: U is every key in order and the stage's centres start at 0;
        // later stages: the GEMM runs on a gathered copy of U and a compact copy
        // of the stage's centres (labels and distances by position in U, as the
        // exact kernel gives them)
        if (t == 0) {
            make_fast(c, k, K, false, c->cent_k, cstride, c->st_m, 0, c->st_labels, c->dmin_k);
        } else if (c->fast_assign && (reinterpret_cast<uintptr_t>(K) & 15u) == 0) {
            const int64_t per = (int64_t)L * (d / 8);
            k_gather_rows_sq<<<dim3((unsigned)((per + 255) / 256), BH), 256, 0, s>>>(K, c->u_idx, c->u_cnt, c->Qp,
                                                                                  c->rowsq_u, L, d);
            AC_NOTE_LAUNCH();
            CK(cudaGetLastError(), "gather stage keys");
            if (make_fast(c, k, c->Qp, false, c->cent_st, (int64_t)m0 * d, c->st_m, 0, c->st_labels, c->dmin_k)) {
                k.fa.rowsq = c->rowsq_u;
                k.fa.nrows = c->u_cnt;
                k.stage_copy = true;
                k.rows = 0;
                for (int h = 0; h < BH; ++h) k.rows += m[h] > 0 ? ucnt[h] : 0;
            }
        }
        CK(run_lloyd(c, k, c->cfg.iters_k, false, s), "k stage lloyd");
        // line 14: d_i = ||k_i - c(k_i)||
        CK(launch_stage_dist(c->dmin_k, c->st_dist, c->u_cnt, c->st_m, L, BH, t == 0 ? c->tau_acc : nullptr, s),
           "stage dist");
        if (t == 0) {
            const int64_t n_total = (int64_t)BH * L;
            if (c->xchg && c->cfg.tau_mode != AC_TAU_ABSOLUTE) {
                ac_status st = exchange_tau(c, s);
                if (st != AC_OK) return st;
            } else if (c->cfg.tau_mode == AC_TAU_MEAN_FACTOR) {
                CK(launch_tau_mean(c->tau_acc, nullptr, n_total, c->cfg.tau_value, c->tau, s), "tau mean");
            } else if (c->cfg.tau_mode == AC_TAU_PERCENTILE) {
                CK(launch_tau_percentile(c->st_dist, c->st_m, L, BH, n_total, (int)c->cfg.tau_value, c->radix,
                                         c->tau, s),
                   "tau percentile");
            } else {
                CK(cudaMemcpyAsync(c->tau, &c->cfg.tau_value, sizeof(float), cudaMemcpyHostToDevice, s), "tau");
            }
        }
        // lines 13-18: drop the keys within tau of their centre from U
        CK(launch_remove(c->st_dist, c->tau, c->u_idx, c->u_idx2, c->u_cnt, c->st_m, c->removed_stage, t, L, BH, s),
           "remove");
        std::swap(c->u_idx, c->u_idx2);
    }
    for (int h = 0; h < BH; ++h) {
        c->h_n_k[h] = nk[h];
        c->h_dense[h] = dense[h];
        c->h_st_m[h] = stages[h];
        c->h_u_cnt[h] = dense[h] ? nk[h] : (stages[h] > 1 ? nk[h] - m_last[h] : 0);
    }
    CK(cudaMemcpyAsync(c->n_k, c->h_n_k, sizeof(int) * BH, cudaMemcpyHostToDevice, s), "n_k");
    CK(cudaMemcpyAsync(c->dense, c->h_dense, BH, cudaMemcpyHostToDevice, s), "dense");
    CK(cudaMemcpyAsync(c->stages, c->h_st_m, sizeof(int) * BH, cudaMemcpyHostToDevice, s), "stages");
    CK(cudaMemcpyAsync(c->fallback_at, c->h_u_cnt, sizeof(int) * BH, cudaMemcpyHostToDevice, s), "fallback");
    CK(cudaStreamSynchronize(s), "stage end sync");  // the staging buffers are reused by the next call
    // line 22: every key to its closest centre among all of C
    Lloyd fin;
    fin.as = AssignArgs{K, nullptr, L, nullptr, nullptr, L, c->cent_k, cstride, nullptr, c->n_k, 0, c->labels_k,
                        c->dmin_k, BH, d};
    make_fast(c, fin, K, false, c->cent_k, cstride, c->n_k, 0, c->labels_k, c->dmin_k);
    CK(assign_pass(c, fin, false, s), "final assign");  // dmin: key statistics
    return AC_OK;
}

// Warm-started step (Sec. 3.2.2 "Efficient initialization"): Lloyd over all
// keys from the previous centres, cluster counts fixed, dense units skipped.
__global__ void k_warm_counts(const int *n_k, const uint8_t *dense, int *ncent, int BH) {
    int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h < BH) ncent[h] = dense[h] ? 0 : n_k[h];
}

ac_status cluster_k_warm(ac_ctx *c, const bf16 *K, cudaStream_t s) {
    const int BH = c->BH, L = c->L, d = c->d;
    const int64_t cstride = (int64_t)c->Ccap * d;
    if (c->fast_assign) CK(launch_row_sqnorm(K, (int64_t)BH * L, d, c->rowsq_k, s), "row norms");
    k_warm_counts<<<(BH + 127) / 128, 128, 0, s>>>(c->n_k, c->dense, c->st_m, BH);
    AC_NOTE_LAUNCH();
    CK(cudaGetLastError(), "warm counts");
    Lloyd k;
    k.as = AssignArgs{K, nullptr, L, nullptr, nullptr, L, c->cent_k, cstride, nullptr, c->st_m, 0, c->labels_k,
                      c->dmin_k, BH, d};
    k.so = SortArgs{c->labels_k, L, nullptr, L, c->n_k, 0, c->Ccap, c->perm_k, c->offs_k, c->Ccap + 1, c->counts_k,
                    c->Ccap, BH, c->sort_scratch};
    k.up = UpdateArgs{K, nullptr, L, nullptr, c->perm_k, c->offs_k, c->Ccap + 1, c->cent_k, cstride, nullptr,
                      c->st_m, 0, BH, d, c->Ccap};
    make_fast(c, k, K, false, c->cent_k, cstride, c->st_m, 0, c->labels_k, c->dmin_k);
    // dmin of the final labels comes from the key statistics
    CK(run_lloyd(c, k, c->cfg.iters_warm, false, s, false), "warm lloyd");
    return AC_OK;
}

// Cluster-order permutation of the keys and the per-cluster statistics.
ac_status key_stats_impl(ac_ctx *c, const bf16 *K, cudaStream_t s) {
    SortArgs so{c->labels_k, c->L, nullptr, c->L, c->n_k, 0, c->Ccap, c->perm_k, c->offs_k, c->Ccap + 1,
                c->counts_k, c->Ccap, c->BH, c->sort_scratch};
    CK(launch_counting_sort(so, s), "k sort");
    StatsArgs st{K, c->L, c->perm_k, c->offs_k, c->Ccap + 1, c->dmin_k, c->n_k, c->Ccap, c->d, c->BH,
                 c->counts_k, c->kmax, c->kmin, c->sse, c->mse, c->comp, c->cent_k, (int64_t)c->Ccap * c->d,
                 c->err, c->st_dist};
    CK(launch_key_stats(st, s), "k stats");
    c->have_k = true;
    return AC_OK;
}

ac_status score_select_impl(ac_ctx *c, int topk, cudaStream_t s) {
    SelectArgs a{c->cent_q, c->kmax, c->kmin, c->counts_k, c->n_k, c->dense, c->offs_k, c->counts_q,
                 c->Cq, c->Ccap, c->d, c->BH, c->L, topk != 0 ? topk : c->cfg.topk,
                 c->score, c->sel, c->ksel, c->ranges, c->nboxes, c->tile_prefix, c->rbox, c->pgoff, c->nrange};
    a.score_mode = c->cfg.score_mode;
    a.cent_k = c->cent_k;
    a.tm_kmax = &c->tm_kmax;
    a.tm_kmin = &c->tm_kmin;
    a.kabs = c->kabs;
    a.err = c->err;
    a.exact_cuda_cores = c->exact_scores;
    a.bound_scale = c->quest_bound_scale;
    if (c->cfg.compensate) {
        a.cbias = c->cbias;
        a.crange = c->crange;
        a.cgroup = c->cgroup;
        a.scale = c->scale;
    }
    CK(launch_score_select(a, s), "score select");
    if (c->cfg.tail_merge) {
        TailMergeArgs t{c->sel, c->ksel, c->dense, c->labels_q, c->perm_q, c->offs_q, c->counts_q, c->counts_k,
                        c->pgoff, c->ranges, c->rbox, c->nrange, c->nboxes, c->perm_qm, c->offs_qm, c->counts_qm,
                        c->tm_scratch, c->tile_prefix, c->Cq, c->Ccap, c->BH, c->cfg.tail_merge, c->L};
        CK(launch_tail_merge(t, s), "tail merge");
    }
    return AC_OK;
}

ac_status sparse_attn_impl(ac_ctx *c, const bf16 *Q, const bf16 *K, const bf16 *V, bf16 *O, cudaStream_t s) {
    // with tail merging the query rows are laid out by group
    const bool tm = c->cfg.tail_merge != 0;
    const int *pq = tm ? c->perm_qm : c->perm_q, *oq = tm ? c->offs_qm : c->offs_q;
    const int *cq = tm ? c->counts_qm : c->counts_q;
    CK(launch_permute_rows(Q, pq, c->Qp, c->L, c->d, c->BH, s), "permute q");
    CK(launch_permute_kv_padded(K, V, c->perm_k, c->labels_k, c->offs_k, c->Ccap + 1, c->pgoff, c->Ccap, c->Kp, c->Vp,
                                c->L, c->Lpad, c->d, c->BH, s),
       "permute k, v");
    if (c->cfg.compensate) {
        // member means of the final key clusters (ascending member order, as the
        // centre update), as bf16 rows of the centroid block
        UpdateArgs uk{K, nullptr, c->L, nullptr, c->perm_k, c->offs_k, c->Ccap + 1, c->kbar, (int64_t)c->Ccap * c->d,
                      nullptr, c->n_k, 0, c->BH, c->d, c->Ccap};
        uk.err = c->err;
        UpdateArgs uv = uk;
        uv.X = V;
        uv.C = c->vbar;
        CK(launch_update(uk, s), "key means");
        CK(launch_update(uv, s), "value means");
        CK(launch_comp_rows(c->kbar, c->vbar, c->n_k, c->Ccap, c->d, c->BH, c->Lpad, c->cgroup, c->Kp, c->Vp, s),
           "centroid rows");
    }
    CK(cudaMemsetAsync(c->counters, 0, 8 * sizeof(unsigned long long), s), "counters");
    AttnArgs a{&c->tm_q, c->tm_kg, c->tm_vg, O, pq, oq, cq, c->tile_prefix, c->ranges,
               c->nboxes, c->nrange, c->rbox, c->L, c->Lpad, c->Cq, c->Ccap, c->BH, c->d,
               (float)(c->scale * 1.4426950408889634), c->err, c->counters};
    if (c->cfg.compensate) {
        a.crange = c->crange;
        a.cbias = c->cbias;
    }
    if (c->timing) CK(cudaEventRecord(c->ev[6], s), "event");
    CK(launch_sparse_attn(a, s), "sparse attention");
    if (c->timing) CK(cudaEventRecord(c->ev[7], s), "event");
    return AC_OK;
}

void free_all(ac_ctx *c) {
    void *dev[] = {c->inv_q, c->labels_q, c->cent_q, c->counts_q, c->perm_q, c->offs_q, c->labels_k, c->dmin_k,
                   c->cent_k, c->n_k, c->dense, c->stages, c->fallback_at, c->removed_stage, c->tau, c->tau_acc, c->counts_k,
                   c->perm_k, c->offs_k, c->kmax, c->kmin, c->sse, c->mse, c->comp, c->u_idx, c->u_idx2,
                   c->u_cnt, c->st_m, c->st_labels, c->st_dist, c->st_perm, c->st_offs, c->st_counts, c->radix,
                   c->score, c->sel, c->ksel, c->ranges, c->nboxes, c->tile_prefix, c->Qp, c->Kp, c->Vp,
                   c->counters, c->hbufQ, c->hbufK, c->hbufV, c->hbufO, c->err, c->chi_q, c->chi_k, c->cn,
                   c->hstat, c->rowsq_k, c->cand, c->amb_list, c->amb_count, c->asg_stats, c->rbox, c->pgoff, c->nrange,
                   c->sort_scratch, c->cnp_k, c->rowsq_u, c->cent_st, c->perm_qm, c->offs_qm, c->counts_qm,
                   c->tm_scratch, c->kabs, c->kbar, c->vbar, c->cbias, c->crange};
    for (void *p : dev)
        if (p) cudaFree(p);
    void *host[] = {c->h_u_cnt, c->h_st_m, c->h_n_k, c->h_dense, c->h_err, c->h_xchg};
    for (void *p : host)
        if (p) cudaFreeHost(p);
    for (auto &e : c->ev)
        if (e) cudaEventDestroy(e);
    for (int b = 0; b < 2; ++b) {
        for (int i = 0; i < 4; ++i)
            if (c->abuf[b][i]) cudaFree(c->abuf[b][i]);
        if (c->ev_in[b]) cudaEventDestroy(c->ev_in[b]);
        if (c->ev_inq[b]) cudaEventDestroy(c->ev_inq[b]);
        if (c->ev_ink[b]) cudaEventDestroy(c->ev_ink[b]);
        if (c->ev_comp[b]) cudaEventDestroy(c->ev_comp[b]);
        if (c->ev_out[b]) cudaEventDestroy(c->ev_out[b]);
    }
    if (c->s_in) cudaStreamDestroy(c->s_in);
    if (c->s_out) cudaStreamDestroy(c->s_out);
}

}  // namespace

void ac::set_static_error(const char *msg) { g_static_msg = msg; }

// ======================================================================== ABI

extern "C" {

const char *ac_last_error_string(const ac_ctx *ctx) { return ctx ? ctx->msg.c_str() : g_static_msg.c_str(); }

ac_status ac_create(const ac_config *cfg, int32_t B, int32_t H, int32_t L, int32_t d, ac_ctx **out) {
    if (!cfg || !out) return AC_ERR_INVALID_ARG;
    *out = nullptr;
    if (B < 1 || H < 1 || L < 1) return AC_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return AC_ERR_UNSUPPORTED;
    if (cfg->Cq < 1 || cfg->Cq > L || cfg->m0 < 1 || cfg->m0 > L || cfg->n_max < 1 || cfg->iters_q < 0 ||
        cfg->iters_k < 0 || cfg->iters_warm < 0 || cfg->tau_mode < 0 || cfg->tau_mode > 2 || cfg->topk == 0 ||
        cfg->stage_rule < 0 || cfg->stage_rule > 1 || (cfg->score_mode != 0 && cfg->score_mode != 1) ||
        cfg->tail_merge < 0 || cfg->tail_merge > 2 || cfg->unit0 < 0 || cfg->compensate < 0 || cfg->compensate > 1 ||
        (cfg->compensate && cfg->tail_merge) || !(cfg->scale >= 0.f) || std::isnan(cfg->tau_value))
        return AC_ERR_INVALID_ARG;
    if ((int64_t)B * H * L >= (int64_t)1 << 31) return AC_ERR_INVALID_ARG;
    if (cfg->tau_mode == AC_TAU_PERCENTILE && (cfg->tau_value < 1.f || cfg->tau_value > 1000.f))
        return AC_ERR_INVALID_ARG;
    if ((int64_t)cfg->n_max + cfg->m0 > 16384) return AC_ERR_INVALID_ARG;
    if (((int64_t)cfg->Cq + 64) * d * 4 > 200 * 1024) return AC_ERR_INVALID_ARG;  // query centroids staged whole

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return AC_ERR_UNSUPPORTED;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return AC_ERR_UNSUPPORTED;
    if (prop.major != 10) return AC_ERR_UNSUPPORTED;

    ac_ctx *c = new (std::nothrow) ac_ctx();
    if (!c) return AC_ERR_WORKSPACE;
    c->cfg = *cfg;
    c->B = B;
    c->H = H;
    c->L = L;
    c->d = d;
    c->BH = B * H;
    c->Cq = cfg->Cq;
    c->Ccap = cfg->n_max + cfg->m0;
    // keys padded per cluster (at most 7 rows each), then the centroid block of
    // ceil(Ccap / 8) groups, then one group that stays zero
    c->Lpad = ((L + 7) & ~7) + 8 * c->Ccap + 16;
    c->cgroup = c->Lpad / 8 - 1 - (c->Ccap + 7) / 8;
    if ((int64_t)c->B * c->H * c->Lpad >= (int64_t)1 << 31) {
        delete c;
        return AC_ERR_INVALID_ARG;
    }
    c->device = dev;
    c->scale = cfg->scale > 0.f ? cfg->scale : 1.0f / std::sqrt((float)d);

    c->num_sms = prop.multiProcessorCount;
    {
        const char *ev = std::getenv("AC_EXACT_ASSIGN");
        c->fast_assign = !(ev && ev[0] == '1');
        const char *es = std::getenv("AC_EXACT_SCORES");
        c->exact_scores = es && es[0] == '1';
        const char *bs = std::getenv("AC_QUEST_BOUND_SCALE");
        c->quest_bound_scale = bs ? std::max(1.0f, (float)std::atof(bs)) : 1.0f;
    }
    c->Cpad_q = (c->Cq + 31) & ~31;
    c->CH_q = std::min(96, c->Cpad_q);  // two-term chunks (c_hi + c_lo) of at most 96 centres
    c->Cpad_k = (c->Ccap + 31) & ~31;
    c->CH_k = std::min(128, c->Cpad_k);
    const size_t BH = c->BH, Lz = L, dz = d, Cq = c->Cq, Cc = c->Ccap, m0 = cfg->m0;
    bool okm = true;
    auto A = [&](cudaError_t e) { okm = okm && e == cudaSuccess; };
    A(dalloc(&c->inv_q, BH * Lz));
    A(dalloc(&c->labels_q, BH * Lz));
    A(dalloc(&c->cent_q, BH * Cq * dz));
    A(dalloc(&c->counts_q, BH * Cq));
    A(dalloc(&c->perm_q, BH * Lz));
    A(dalloc(&c->offs_q, BH * (Cq + 1)));
    A(dalloc(&c->labels_k, BH * Lz));
    A(dalloc(&c->dmin_k, BH * Lz));
    A(dalloc(&c->cent_k, BH * Cc * dz));
    A(dalloc(&c->n_k, BH));
    A(dalloc(&c->dense, BH));
    A(dalloc(&c->stages, BH));
    A(dalloc(&c->fallback_at, BH));
    A(dalloc(&c->removed_stage, BH * Lz));
    A(dalloc(&c->tau, 1));
    A(dalloc(&c->tau_acc, 1));
    A(dalloc(&c->counts_k, BH * Cc));
    A(dalloc(&c->perm_k, BH * Lz));
    A(dalloc(&c->offs_k, BH * (Cc + 1)));
    A(dalloc(&c->kmax, BH * Cc * dz));
    A(dalloc(&c->kmin, BH * Cc * dz));
    A(dalloc(&c->sse, BH * Cc));
    A(dalloc(&c->mse, BH));
    A(dalloc(&c->comp, BH));
    A(dalloc(&c->u_idx, BH * Lz));
    A(dalloc(&c->u_idx2, BH * Lz));
    A(dalloc(&c->u_cnt, BH));
    A(dalloc(&c->st_m, BH));
    A(dalloc(&c->st_labels, BH * Lz));
    A(dalloc(&c->st_dist, BH * Lz));
    A(dalloc(&c->st_perm, BH * Lz));
    A(dalloc(&c->st_offs, BH * (m0 + 1)));
    A(dalloc(&c->st_counts, BH * m0));
    A(dalloc(&c->radix, 260));
    A(dalloc(&c->sort_scratch, BH * 129 * std::max(Cc, Cq)));  // chunk histograms + label totals
    A(dalloc(&c->score, BH * Cq * Cc));
    A(dalloc(&c->kabs, BH * Cc));
    A(dalloc(&c->sel, BH * Cq * Cc));
    A(dalloc(&c->ksel, BH));
    A(dalloc(&c->ranges, BH * Cq * Cc));
    A(dalloc(&c->nboxes, BH * Cq));
    A(dalloc(&c->rbox, BH * Cq * (Cc + 1)));
    A(dalloc(&c->tile_prefix, BH * Cq + 1));
    A(dalloc(&c->chi_q, 2 * BH * c->Cpad_q * dz));
    A(dalloc(&c->chi_k, BH * c->Cpad_k * dz));
    A(dalloc(&c->cnp_k, BH * c->Cpad_k * 16));
    A(dalloc(&c->cn, BH * std::max(c->Cpad_q, c->Cpad_k)));
    A(dalloc(&c->hstat, 2 * BH));
    A(dalloc(&c->rowsq_k, BH * Lz));
    A(dalloc(&c->rowsq_u, BH * Lz));
    if (cfg->compensate) {
        A(dalloc(&c->kbar, BH * Cc * dz));
        A(dalloc(&c->vbar, BH * Cc * dz));
        A(dalloc(&c->cbias, BH * Cq * Cc));
        A(dalloc(&c->crange, BH * Cq));
    }
    if (cfg->tail_merge) {
        A(dalloc(&c->perm_qm, BH * Lz));
        A(dalloc(&c->offs_qm, BH * (Cq + 1)));
        A(dalloc(&c->counts_qm, BH * Cq));
        A(dalloc(&c->tm_scratch, 4 * BH * Cq));
    }
    A(dalloc(&c->cent_st, BH * (size_t)m0 * dz));
    A(dalloc(&c->cand, BH * Lz));
    A(dalloc(&c->amb_list, BH * Lz));
    A(dalloc(&c->amb_count, 2));
    A(dalloc(&c->asg_stats, 2));
    A(dalloc(&c->Qp, BH * Lz * dz));
    A(dalloc(&c->Kp, BH * (size_t)c->Lpad * dz));
    A(dalloc(&c->Vp, BH * (size_t)c->Lpad * dz));
    A(dalloc(&c->pgoff, BH * Cc));
    A(dalloc(&c->nrange, BH * Cq));
    A(dalloc(&c->counters, 8));
    A(dalloc(&c->err, 1));
    A(cudaMallocHost(&c->h_u_cnt, BH * sizeof(int)));
    A(cudaMallocHost(&c->h_st_m, BH * sizeof(int)));
    A(cudaMallocHost(&c->h_n_k, BH * sizeof(int)));
    A(cudaMallocHost(&c->h_dense, BH));
    A(cudaMallocHost(&c->h_err, sizeof(uint32_t)));
    A(cudaMallocHost(&c->h_xchg, 256 * sizeof(uint64_t) + 256 * sizeof(uint32_t)));
    for (auto &e : c->ev) A(cudaEventCreate(&e));
    if (!okm) {
        free_all(c);
        delete c;
        cudaGetLastError();
        return AC_ERR_WORKSPACE;
    }
    if (cudaMemset(c->err, 0, sizeof(uint32_t)) != cudaSuccess ||
        cudaMemset(c->asg_stats, 0, 2 * sizeof(unsigned long long)) != cudaSuccess ||
        cudaMemset(c->dense, 0, BH) != cudaSuccess || cudaMemset(c->n_k, 0, BH * sizeof(int)) != cudaSuccess ||
        // padding rows of Kp / Vp are read (and masked) by the attention: keep them finite
        cudaMemset(c->Kp, 0, BH * (size_t)c->Lpad * dz * sizeof(bf16)) != cudaSuccess ||
        cudaMemset(c->Vp, 0, BH * (size_t)c->Lpad * dz * sizeof(bf16)) != cudaSuccess ||
        // an empty cluster's member mean is never written: keep it finite
        (c->kbar && cudaMemset(c->kbar, 0, BH * Cc * dz * sizeof(float)) != cudaSuccess) ||
        (c->vbar && cudaMemset(c->vbar, 0, BH * Cc * dz * sizeof(float)) != cudaSuccess)) {
        free_all(c);
        delete c;
        return AC_ERR_CUDA;
    }
    const int64_t rows = (int64_t)BH * L;
    bool maps_ok = make_tmap(c, &c->tm_q, c->Qp, rows, d, 128) == AC_OK;
    for (int i = 0; i < 4 && maps_ok; ++i)
        maps_ok = make_tmap_kv(c, &c->tm_kg[i], c->Kp, (int64_t)BH * c->Lpad / 8, d, 1 << i) == AC_OK &&
                  make_tmap_kv(c, &c->tm_vg[i], c->Vp, (int64_t)BH * c->Lpad / 8, d, 1 << i) == AC_OK;
    if (!maps_ok ||
        make_tmap(c, &c->tm_chi_q, c->chi_q, (int64_t)2 * BH * c->Cpad_q, d, c->CH_q) != AC_OK ||
        make_tmap(c, &c->tm_chi_k, c->chi_k, (int64_t)BH * c->Cpad_k, d, c->CH_k) != AC_OK ||
        make_tmap_plain16(c, &c->tm_cnp_k, c->cnp_k, (int64_t)BH * c->Cpad_k, c->CH_k) != AC_OK ||
        make_tmap(c, &c->tm_kmax, c->kmax, (int64_t)BH * c->Ccap, d, 64) != AC_OK ||
        make_tmap(c, &c->tm_kmin, c->kmin, (int64_t)BH * c->Ccap, d, 64) != AC_OK) {
        free_all(c);
        delete c;
        return AC_ERR_CUDA;
    }
    *out = c;
    return AC_OK;
}

ac_status ac_destroy(ac_ctx *c) {
    if (!c) return AC_ERR_INVALID_ARG;
    cudaDeviceSynchronize();
    free_all(c);
    delete c;
    return AC_OK;
}

ac_status ac_cluster_q(ac_ctx *c, const uint16_t *Q, const float *init, int32_t iters, int32_t *labels_out,
                       float *cent_out, void *stream) {
    if (!c || !Q) return fail(c, AC_ERR_INVALID_ARG, "ac_cluster_q: NULL argument");
    cudaStream_t s = (cudaStream_t)stream;
    const int T = iters >= 0 ? iters : (init ? c->cfg.iters_warm : c->cfg.iters_q);
    ac_status st = cluster_q_impl(c, reinterpret_cast<const bf16 *>(Q), init, T, s);
    if (st != AC_OK) return st;
    if (labels_out)
        CK(cudaMemcpyAsync(labels_out, c->labels_q, sizeof(int) * (size_t)c->BH * c->L, cudaMemcpyDeviceToDevice, s),
           "labels out");
    if (cent_out)
        CK(cudaMemcpyAsync(cent_out, c->cent_q, sizeof(float) * (size_t)c->BH * c->Cq * c->d,
                           cudaMemcpyDeviceToDevice, s),
           "centres out");
    return check_dev_err(c, s);
}

ac_status ac_cluster_k_multistage(ac_ctx *c, const uint16_t *K, const float *warm_cent, const int32_t *warm_n_k,
                                  const uint8_t *warm_dense, int32_t *labels_out, float *cent_out, int32_t *n_k_out,
                                  uint8_t *dense_out, float *comp_out, void *stream) {
    if (!c || !K) return fail(c, AC_ERR_INVALID_ARG, "ac_cluster_k_multistage: NULL argument");
    if ((warm_cent == nullptr) != (warm_n_k == nullptr))
        return fail(c, AC_ERR_INVALID_ARG, "warm start needs both centres and counts");
    cudaStream_t s = (cudaStream_t)stream;
    const bf16 *Kb = reinterpret_cast<const bf16 *>(K);
    const size_t BH = c->BH;
    ac_status st;
    if (warm_cent) {
        if (warm_cent != c->cent_k)
            CK(cudaMemcpyAsync(c->cent_k, warm_cent, sizeof(float) * BH * c->Ccap * c->d, cudaMemcpyDeviceToDevice, s),
               "warm centres");
        if (warm_n_k != c->n_k) {
            // the counts index the centre arrays: check them before any kernel uses them
            std::vector<int32_t> nk(BH);
            CK(cudaMemcpyAsync(nk.data(), warm_n_k, sizeof(int) * BH, cudaMemcpyDeviceToHost, s), "warm counts");
            CK(cudaStreamSynchronize(s), "warm counts");
            for (size_t h = 0; h < BH; ++h)
                if (nk[h] < 0 || nk[h] > c->Ccap)
                    return fail(c, AC_ERR_INVALID_ARG, "warm cluster count out of range [0, n_max + m0]");
            CK(cudaMemcpyAsync(c->n_k, warm_n_k, sizeof(int) * BH, cudaMemcpyDeviceToDevice, s), "warm counts");
        }
        if (warm_dense) {
            if (warm_dense != c->dense)
                CK(cudaMemcpyAsync(c->dense, warm_dense, BH, cudaMemcpyDeviceToDevice, s), "warm dense");
        } else {
            CK(cudaMemsetAsync(c->dense, 0, BH, s), "warm dense");
        }
        st = cluster_k_warm(c, Kb, s);
    } else {
        st = cluster_k_step0(c, Kb, s);
    }
    if (st != AC_OK) return st;
    if ((st = key_stats_impl(c, Kb, s)) != AC_OK) return st;
    if (labels_out) CK(cudaMemcpyAsync(labels_out, c->labels_k, sizeof(int) * BH * c->L, cudaMemcpyDeviceToDevice, s), "out");
    if (cent_out)
        CK(cudaMemcpyAsync(cent_out, c->cent_k, sizeof(float) * BH * c->Ccap * c->d, cudaMemcpyDeviceToDevice, s), "out");
    if (n_k_out) CK(cudaMemcpyAsync(n_k_out, c->n_k, sizeof(int) * BH, cudaMemcpyDeviceToDevice, s), "out");
    if (dense_out) CK(cudaMemcpyAsync(dense_out, c->dense, BH, cudaMemcpyDeviceToDevice, s), "out");
    if (comp_out) CK(cudaMemcpyAsync(comp_out, c->comp, sizeof(float) * BH, cudaMemcpyDeviceToDevice, s), "out");
    c->have_state = c->have_q;
    return check_dev_err(c, s);
}

ac_status ac_score_select(ac_ctx *c, int32_t topk, int32_t *sel_out, int32_t *k_out, void *stream) {
    if (!c) return AC_ERR_INVALID_ARG;
    if (!c->have_q || !c->have_k) return fail(c, AC_ERR_STATE, "ac_score_select before clustering");
    cudaStream_t s = (cudaStream_t)stream;
    ac_status st = score_select_impl(c, topk, s);
    if (st != AC_OK) return st;
    if (sel_out)
        CK(cudaMemcpyAsync(sel_out, c->sel, sizeof(int) * (size_t)c->BH * c->Cq * c->Ccap, cudaMemcpyDeviceToDevice,
                           s),
           "sel out");
    if (k_out) CK(cudaMemcpyAsync(k_out, c->ksel, sizeof(int) * (size_t)c->BH, cudaMemcpyDeviceToDevice, s), "k out");
    return AC_OK;
}

ac_status ac_sparse_attn(ac_ctx *c, const uint16_t *Q, const uint16_t *K, const uint16_t *V, uint16_t *O,
                         void *stream) {
    if (!c || !Q || !K || !V || !O) return fail(c, AC_ERR_INVALID_ARG, "ac_sparse_attn: NULL argument");
    if (!c->have_q || !c->have_k) return fail(c, AC_ERR_STATE, "ac_sparse_attn before clustering");
    return sparse_attn_impl(c, reinterpret_cast<const bf16 *>(Q), reinterpret_cast<const bf16 *>(K),
                            reinterpret_cast<const bf16 *>(V), reinterpret_cast<bf16 *>(O), (cudaStream_t)stream);
}

namespace {
// The layer's steps on stream s; each of wq, wk, wv (nullable) is an event the
// stream waits for before the first step that reads Q, K or V respectively.
ac_status layer_steps(ac_ctx *c, const uint16_t *Q, const uint16_t *K, const uint16_t *V, uint16_t *O, int32_t warm,
                      ac_stage_times *times, cudaStream_t s, cudaEvent_t wq, cudaEvent_t wk, cudaEvent_t wv) {
    const bf16 *Qb = reinterpret_cast<const bf16 *>(Q), *Kb = reinterpret_cast<const bf16 *>(K),
               *Vb = reinterpret_cast<const bf16 *>(V);
    ac_status st;
    c->timing = times != nullptr;
    if (times) CK(cudaEventRecord(c->ev[0], s), "event");
    if (wq) CK(cudaStreamWaitEvent(s, wq, 0), "wait Q");
    st = cluster_q_impl(c, Qb, warm ? c->cent_q : nullptr, warm ? c->cfg.iters_warm : c->cfg.iters_q, s);
    if (st != AC_OK) return st;
    if (times) CK(cudaEventRecord(c->ev[1], s), "event");
    if (wk) CK(cudaStreamWaitEvent(s, wk, 0), "wait K");
    st = warm ? cluster_k_warm(c, Kb, s) : cluster_k_step0(c, Kb, s);
    if (st != AC_OK) return st;
    if (times) CK(cudaEventRecord(c->ev[2], s), "event");
    if ((st = key_stats_impl(c, Kb, s)) != AC_OK) return st;
    if (times) CK(cudaEventRecord(c->ev[3], s), "event");
    if ((st = score_select_impl(c, 0, s)) != AC_OK) return st;
    if (times) CK(cudaEventRecord(c->ev[4], s), "event");
    if (wv) CK(cudaStreamWaitEvent(s, wv, 0), "wait V");
    if ((st = sparse_attn_impl(c, Qb, Kb, Vb, reinterpret_cast<bf16 *>(O), s)) != AC_OK) return st;
    return AC_OK;
}
}  // namespace

ac_status ac_layer_forward(ac_ctx *c, const uint16_t *Q, const uint16_t *K, const uint16_t *V, uint16_t *O,
                           int32_t warm, ac_stage_times *times, void *stream) {
    if (!c || !Q || !K || !V || !O) return fail(c, AC_ERR_INVALID_ARG, "ac_layer_forward: NULL argument");
    if (warm && !c->have_state) return fail(c, AC_ERR_STATE, "warm step before any step 0");
    cudaStream_t s = (cudaStream_t)stream;
    ac_status st = layer_steps(c, Q, K, V, O, warm, times, s, nullptr, nullptr, nullptr);
    if (st != AC_OK) return st;
    if (times) CK(cudaEventRecord(c->ev[5], s), "event");
    c->have_state = true;
    if (times) {
        CK(cudaEventSynchronize(c->ev[5]), "event sync");
        float ms[5];
        for (int i = 0; i < 5; ++i) CK(cudaEventElapsedTime(&ms[i], c->ev[i], c->ev[i + 1]), "elapsed");
        times->q_cluster_ms = ms[0];
        times->k_cluster_ms = ms[1];
        times->stats_sort_ms = ms[2];
        times->score_select_ms = ms[3];
        times->attention_ms = ms[4];
        CK(cudaEventElapsedTime(&times->attn_kernel_ms, c->ev[6], c->ev[7]), "elapsed");
        CK(cudaEventElapsedTime(&times->total_ms, c->ev[0], c->ev[5]), "elapsed");
        c->timing = false;
        return check_dev_err(c, s);
    }
    return AC_OK;
}

ac_status ac_layer_forward_host(ac_ctx *c, const uint16_t *hQ, const uint16_t *hK, const uint16_t *hV,
                                uint16_t *hO, int32_t warm, void *stream) {
    if (!c || !hQ || !hK || !hV || !hO) return fail(c, AC_ERR_INVALID_ARG, "ac_layer_forward_host: NULL argument");
    cudaStream_t s = (cudaStream_t)stream;
    const size_t n = (size_t)c->BH * c->L * c->d;
    if (!c->hbufQ) {
        if (dalloc(&c->hbufQ, n) != cudaSuccess || dalloc(&c->hbufK, n) != cudaSuccess ||
            dalloc(&c->hbufV, n) != cudaSuccess || dalloc(&c->hbufO, n) != cudaSuccess) {
            cudaGetLastError();
            return fail(c, AC_ERR_WORKSPACE, "host-buffer staging allocation failed");
        }
    }
    CK(cudaMemcpyAsync(c->hbufQ, hQ, n * 2, cudaMemcpyHostToDevice, s), "h2d Q");
    CK(cudaMemcpyAsync(c->hbufK, hK, n * 2, cudaMemcpyHostToDevice, s), "h2d K");
    CK(cudaMemcpyAsync(c->hbufV, hV, n * 2, cudaMemcpyHostToDevice, s), "h2d V");
    ac_status st = ac_layer_forward(c, c->hbufQ, c->hbufK, c->hbufV, c->hbufO, warm, nullptr, stream);
    if (st != AC_OK) return st;
    CK(cudaMemcpyAsync(hO, c->hbufO, n * 2, cudaMemcpyDeviceToHost, s), "d2h O");
    return check_dev_err(c, s);
}

ac_status ac_get_tensor(ac_ctx *c, int32_t which, void **ptr, int64_t shape[4]) {
    if (!c || !ptr || !shape) return AC_ERR_INVALID_ARG;
    const int64_t BH = c->BH, L = c->L, d = c->d, Cq = c->Cq, Cc = c->Ccap;
    int64_t s0 = 1, s1 = 1, s2 = 1;
    void *p = nullptr;
    switch (which) {
        case AC_T_INV_NORM_Q: p = c->inv_q; s0 = BH; s1 = L; break;
        case AC_T_LABELS_Q: p = c->labels_q; s0 = BH; s1 = L; break;
        case AC_T_CENT_Q: p = c->cent_q; s0 = BH; s1 = Cq; s2 = d; break;
        case AC_T_COUNTS_Q: p = c->counts_q; s0 = BH; s1 = Cq; break;
        case AC_T_PERM_Q: p = c->perm_q; s0 = BH; s1 = L; break;
        case AC_T_OFFS_Q: p = c->offs_q; s0 = BH; s1 = Cq + 1; break;
        case AC_T_LABELS_K: p = c->labels_k; s0 = BH; s1 = L; break;
        case AC_T_DMIN_K: p = c->dmin_k; s0 = BH; s1 = L; break;
        case AC_T_CENT_K: p = c->cent_k; s0 = BH; s1 = Cc; s2 = d; break;
        case AC_T_N_K: p = c->n_k; s0 = BH; break;
        case AC_T_DENSE: p = c->dense; s0 = BH; break;
        case AC_T_COUNTS_K: p = c->counts_k; s0 = BH; s1 = Cc; break;
        case AC_T_KMAX: p = c->kmax; s0 = BH; s1 = Cc; s2 = d; break;
        case AC_T_KMIN: p = c->kmin; s0 = BH; s1 = Cc; s2 = d; break;
        case AC_T_SSE: p = c->sse; s0 = BH; s1 = Cc; break;
        case AC_T_COMP: p = c->comp; s0 = BH; break;
        case AC_T_PERM_K: p = c->perm_k; s0 = BH; s1 = L; break;
        case AC_T_OFFS_K: p = c->offs_k; s0 = BH; s1 = Cc + 1; break;
        case AC_T_SCORE: p = c->score; s0 = BH; s1 = Cq; s2 = Cc; break;
        case AC_T_SEL: p = c->sel; s0 = BH; s1 = Cq; s2 = Cc; break;
        case AC_T_KSEL: p = c->ksel; s0 = BH; break;
        case AC_T_TAU: p = c->tau; s0 = 1; break;
        case AC_T_STAGES: p = c->stages; s0 = BH; break;
        case AC_T_REMOVED_STAGE: p = c->removed_stage; s0 = BH; s1 = L; break;
        case AC_T_MSE: p = c->mse; s0 = BH; break;
        case AC_T_FALLBACK_AT: p = c->fallback_at; s0 = BH; break;
        default: return fail(c, AC_ERR_INVALID_ARG, "unknown tensor id");
    }
    *ptr = p;
    shape[0] = s0;
    shape[1] = s1;
    shape[2] = s2;
    shape[3] = 1;
    return AC_OK;
}

ac_status ac_get_launch_count(int64_t *out) {
    if (!out) return AC_ERR_INVALID_ARG;
    *out = (int64_t)g_launches.load(std::memory_order_relaxed);
    return AC_OK;
}

ac_status ac_calibrate_n_max(const int32_t *fallback_at, int64_t n, float dense_frac, int32_t *n_max) {
    if (!fallback_at || !n_max || n < 1 || !(dense_frac >= 0.f && dense_frac <= 1.f)) return AC_ERR_INVALID_ARG;
    std::vector<int32_t> v(fallback_at, fallback_at + n);
    std::sort(v.begin(), v.end(), std::greater<int32_t>());
    // ceil(dense_frac * n); 1e-4 forgives the rounding of dense_frac to fp32 (0.1f * 10 > 1)
    const int64_t k = std::max<int64_t>(0, (int64_t)std::ceil((double)dense_frac * (double)n - 1e-4));
    if (k == 0) {
        *n_max = v[0] + 1;
        return AC_OK;
    }
    if (v[0] <= 0) return AC_ERR_INVALID_ARG;  // no unit ran more than one stage: none can fall back
    int32_t t = v[k - 1];
    if (t <= 0) {  // fewer than k multi-stage units: all of them
        t = v[0];
        for (int64_t i = 0; i < n; ++i)
            if (v[i] > 0) t = v[i];
    }
    *n_max = t;
    return AC_OK;
}

ac_status ac_set_tau_exchange(ac_ctx *c, ac_sum_u64_fn fn, void *user) {
    if (!c) return AC_ERR_INVALID_ARG;
    c->xchg = fn;
    c->xchg_user = user;
    return AC_OK;
}

ac_status ac_tau_mean_from_sums(float factor, uint64_t fixed_sum, uint64_t n, float *tau) {
    if (!tau || n == 0) return AC_ERR_INVALID_ARG;
    // the operations of k_tau_mean: fp64, round to nearest, then fp32
    const double mean = ((double)fixed_sum / 16777216.0) / (double)n;
    *tau = (float)((double)factor * mean);
    return AC_OK;
}

ac_status ac_tau_radix_pick(const uint64_t *hist, int32_t shift, uint32_t *state) {
    if (!hist || !state || shift < 0 || shift > 24 || (shift & 7)) return AC_ERR_INVALID_ARG;
    // the digit of the rank-th smallest (0-based) among the matching distances
    const uint64_t rank = state[2];
    uint64_t cum = 0;
    int dg = -1;
    for (int i = 0; i < 256; ++i) {
        if (cum + hist[i] > rank) {
            dg = i;
            break;
        }
        cum += hist[i];
    }
    if (dg < 0) return AC_ERR_INVALID_ARG;
    state[2] = (uint32_t)(rank - cum);
    state[0] |= (uint32_t)dg << shift;
    state[1] |= 255u << shift;
    return AC_OK;
}

// One thread waits, with the same bounded loop as the pipelined kernels, on
// the first phase of an mbarrier that expects one arrival which never comes;
// when the limit runs out it records DEV_ERR_TIMEOUT and the CTA returns.
__global__ void k_wait_check(uint32_t *err, uint64_t limit_ns) {
    __shared__ alignas(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
        if (!mbar_wait_for(smem_u32(&bar), 0, limit_ns)) set_err(err, DEV_ERR_TIMEOUT);
    }
}

ac_status ac_check_wait_timeout(ac_ctx *c, int32_t limit_us, void *stream) {
    if (!c) return AC_ERR_INVALID_ARG;
    if (limit_us < 1 || limit_us > 2000000)
        return fail(c, AC_ERR_INVALID_ARG, "ac_check_wait_timeout: limit_us outside 1 .. 2,000,000");
    k_wait_check<<<1, 32, 0, (cudaStream_t)stream>>>(c->err, (uint64_t)limit_us * 1000ull);
    AC_NOTE_LAUNCH();
    CK(cudaGetLastError(), "wait check launch");
    return AC_OK;
}

ac_status ac_synchronize(ac_ctx *c, void *stream) {
    if (!c) return AC_ERR_INVALID_ARG;
    ac_status st = ac_join(c, stream);
    if (st != AC_OK) return st;
    return check_dev_err(c, (cudaStream_t)stream);
}

ac_status ac_join(ac_ctx *c, void *stream) {
    if (!c) return AC_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    for (int b = 0; b < 2; ++b)
        if (c->ev_out[b]) CK(cudaStreamWaitEvent(s, c->ev_out[b], 0), "join");
    return AC_OK;
}

// Call n uses staging set n % 2.  Inputs of call n are copied on s_in once
// call n - 2 (same set) has finished its layer; the layer runs on the caller's
// stream once those inputs have landed and call n - 2's output copy has left
// the set; the output is copied on s_out once the layer is done.  So call n's
// input copy overlaps call n - 1's layer, and its output copy call n + 1's.
ac_status ac_layer_forward_host_async(ac_ctx *c, const uint16_t *hQ, const uint16_t *hK, const uint16_t *hV,
                                      uint16_t *hO, int32_t warm, void *stream) {
    if (!c || !hQ || !hK || !hV || !hO)
        return fail(c, AC_ERR_INVALID_ARG, "ac_layer_forward_host_async: NULL argument");
    if (warm && !c->have_state) return fail(c, AC_ERR_STATE, "warm step before any step 0");
    cudaStream_t s = (cudaStream_t)stream;
    const size_t n = (size_t)c->BH * c->L * c->d;
    if (!c->s_in) {
        for (int b = 0; b < 2; ++b)
            for (int i = 0; i < 4; ++i)
                if (dalloc(&c->abuf[b][i], n) != cudaSuccess) {
                    cudaGetLastError();
                    return fail(c, AC_ERR_WORKSPACE, "host-buffer staging allocation failed");
                }
        for (int b = 0; b < 2; ++b) {
            CK(cudaEventCreateWithFlags(&c->ev_in[b], cudaEventDisableTiming), "event");
            CK(cudaEventCreateWithFlags(&c->ev_inq[b], cudaEventDisableTiming), "event");
            CK(cudaEventCreateWithFlags(&c->ev_ink[b], cudaEventDisableTiming), "event");
            CK(cudaEventCreateWithFlags(&c->ev_comp[b], cudaEventDisableTiming), "event");
            CK(cudaEventCreateWithFlags(&c->ev_out[b], cudaEventDisableTiming), "event");
        }
        CK(cudaStreamCreateWithFlags(&c->s_in, cudaStreamNonBlocking), "stream");
        CK(cudaStreamCreateWithFlags(&c->s_out, cudaStreamNonBlocking), "stream");
    }
    const int b = (int)(c->async_calls & 1);
    uint16_t **buf = c->abuf[b];
    if (c->async_calls >= 2) CK(cudaStreamWaitEvent(c->s_in, c->ev_comp[b], 0), "wait layer");
    // Q, K and V land one after the other; the layer starts on Q as soon as it
    // has landed (the query clustering overlaps the copies of K and V)
    CK(cudaMemcpyAsync(buf[0], hQ, n * 2, cudaMemcpyHostToDevice, c->s_in), "h2d Q");
    CK(cudaEventRecord(c->ev_inq[b], c->s_in), "event");
    CK(cudaMemcpyAsync(buf[1], hK, n * 2, cudaMemcpyHostToDevice, c->s_in), "h2d K");
    CK(cudaEventRecord(c->ev_ink[b], c->s_in), "event");
    CK(cudaMemcpyAsync(buf[2], hV, n * 2, cudaMemcpyHostToDevice, c->s_in), "h2d V");
    CK(cudaEventRecord(c->ev_in[b], c->s_in), "event");
    if (c->async_calls >= 2) CK(cudaStreamWaitEvent(s, c->ev_out[b], 0), "wait output copy");
    ++c->async_calls;
    ac_status st = layer_steps(c, buf[0], buf[1], buf[2], buf[3], warm, nullptr, s, c->ev_inq[b], c->ev_ink[b],
                               c->ev_in[b]);
    if (st != AC_OK) {
        // Kernels of this call may already be enqueued and read set b: the
        // set's events must order its next use after them, as on success.
        if (cudaEventRecord(c->ev_comp[b], s) == cudaSuccess &&
            cudaStreamWaitEvent(c->s_out, c->ev_comp[b], 0) == cudaSuccess)
            cudaEventRecord(c->ev_out[b], c->s_out);
        return st;
    }
    c->have_state = true;
    CK(cudaEventRecord(c->ev_comp[b], s), "event");
    CK(cudaStreamWaitEvent(c->s_out, c->ev_comp[b], 0), "wait layer");
    CK(cudaMemcpyAsync(hO, buf[3], n * 2, cudaMemcpyDeviceToHost, c->s_out), "d2h O");
    CK(cudaEventRecord(c->ev_out[b], c->s_out), "event");
    return AC_OK;
}

ac_status ac_get_assign_counters(ac_ctx *c, ac_assign_counters *out, int32_t reset) {
    if (!c || !out) return AC_ERR_INVALID_ARG;
    unsigned long long h[2];
    CK(cudaDeviceSynchronize(), "sync");
    CK(cudaMemcpy(h, c->asg_stats, sizeof(h), cudaMemcpyDeviceToHost), "assign counters");
    out->tensor_passes = c->n_fast;
    out->exact_passes = c->n_exact;
    out->rows = c->n_fast_rows;
    out->uncertain_rows = (int64_t)h[0];
    out->full_rescore_rows = (int64_t)h[1];
    if (reset) {
        CK(cudaMemset(c->asg_stats, 0, sizeof(h)), "assign counters reset");
        c->n_fast = c->n_exact = c->n_fast_rows = 0;
    }
    return AC_OK;
}

ac_status ac_get_attn_counters(ac_ctx *c, ac_attn_counters *out) {
    if (!c || !out) return AC_ERR_INVALID_ARG;
    unsigned long long h[8];
    CK(cudaDeviceSynchronize(), "sync");
    CK(cudaMemcpy(h, c->counters, sizeof(h), cudaMemcpyDeviceToHost), "counters");
    std::vector<uint8_t> dn(c->BH);
    CK(cudaMemcpy(dn.data(), c->dense, c->BH, cudaMemcpyDeviceToHost), "dense");
    out->kept_pairs = (int64_t)h[0];
    out->computed_pairs = (int64_t)h[1];
    out->tiles = (int64_t)h[2];
    out->wait_failure = (int64_t)h[4];
    out->dense_heads = 0;
    for (uint8_t v : dn) out->dense_heads += v ? 1 : 0;
    return AC_OK;
}

// State layout: magic, B, H, L, d, Cq, Ccap, then cent_q, cent_k, n_k, dense,
// labels_k, dmin_k.
ac_status ac_state_export(ac_ctx *c, void *host_buf, int64_t *bytes) {
    if (!c || !bytes) return AC_ERR_INVALID_ARG;
    const size_t BH = c->BH;
    const size_t sz_q = BH * c->Cq * c->d * 4, sz_k = BH * c->Ccap * c->d * 4, sz_n = BH * 4, sz_f = BH,
                 sz_l = BH * c->L * 4;
    const size_t total = 8 * 8 + sz_q + sz_k + sz_n + sz_f + 2 * sz_l;
    if (!host_buf) {
        *bytes = (int64_t)total;
        return AC_OK;
    }
    if (*bytes < (int64_t)total) return fail(c, AC_ERR_INVALID_ARG, "state buffer too small");
    if (!c->have_state) return fail(c, AC_ERR_STATE, "no state to export");
    CK(cudaDeviceSynchronize(), "sync");
    int64_t *hd = reinterpret_cast<int64_t *>(host_buf);
    hd[0] = 0x41435354415445LL;
    hd[1] = c->B;
    hd[2] = c->H;
    hd[3] = c->L;
    hd[4] = c->d;
    hd[5] = c->Cq;
    hd[6] = c->Ccap;
    hd[7] = 0;
    uint8_t *p = reinterpret_cast<uint8_t *>(host_buf) + 64;
    CK(cudaMemcpy(p, c->cent_q, sz_q, cudaMemcpyDeviceToHost), "export");
    p += sz_q;
    CK(cudaMemcpy(p, c->cent_k, sz_k, cudaMemcpyDeviceToHost), "export");
    p += sz_k;
    CK(cudaMemcpy(p, c->n_k, sz_n, cudaMemcpyDeviceToHost), "export");
    p += sz_n;
    CK(cudaMemcpy(p, c->dense, sz_f, cudaMemcpyDeviceToHost), "export");
    p += sz_f;
    CK(cudaMemcpy(p, c->labels_k, sz_l, cudaMemcpyDeviceToHost), "export");
    p += sz_l;
    CK(cudaMemcpy(p, c->dmin_k, sz_l, cudaMemcpyDeviceToHost), "export");
    *bytes = (int64_t)total;
    return AC_OK;
}

ac_status ac_state_import(ac_ctx *c, const void *host_buf, int64_t bytes) {
    if (!c || !host_buf) return AC_ERR_INVALID_ARG;
    int64_t need = 0;
    ac_state_export(c, nullptr, &need);
    if (bytes < need) return fail(c, AC_ERR_INVALID_ARG, "state buffer too small");
    const int64_t *hd = reinterpret_cast<const int64_t *>(host_buf);
    if (hd[0] != 0x41435354415445LL || hd[1] != c->B || hd[2] != c->H || hd[3] != c->L || hd[4] != c->d ||
        hd[5] != c->Cq || hd[6] != c->Ccap)
        return fail(c, AC_ERR_INVALID_ARG, "state does not match this context");
    const size_t BH = c->BH;
    const size_t sz_q = BH * c->Cq * c->d * 4, sz_k = BH * c->Ccap * c->d * 4, sz_n = BH * 4, sz_f = BH,
                 sz_l = BH * c->L * 4;
    {
        const int32_t *nk = reinterpret_cast<const int32_t *>(reinterpret_cast<const uint8_t *>(host_buf) + 64 +
                                                              sz_q + sz_k);
        for (size_t h = 0; h < BH; ++h)
            if (nk[h] < 0 || nk[h] > c->Ccap) return fail(c, AC_ERR_INVALID_ARG, "state: cluster count out of range");
    }
    CK(cudaDeviceSynchronize(), "sync");
    const uint8_t *p = reinterpret_cast<const uint8_t *>(host_buf) + 64;
    CK(cudaMemcpy(c->cent_q, p, sz_q, cudaMemcpyHostToDevice), "import");
    p += sz_q;
    CK(cudaMemcpy(c->cent_k, p, sz_k, cudaMemcpyHostToDevice), "import");
    p += sz_k;
    CK(cudaMemcpy(c->n_k, p, sz_n, cudaMemcpyHostToDevice), "import");
    p += sz_n;
    CK(cudaMemcpy(c->dense, p, sz_f, cudaMemcpyHostToDevice), "import");
    p += sz_f;
    CK(cudaMemcpy(c->labels_k, p, sz_l, cudaMemcpyHostToDevice), "import");
    p += sz_l;
    CK(cudaMemcpy(c->dmin_k, p, sz_l, cudaMemcpyHostToDevice), "import");
    c->have_state = true;
    c->have_q = true;
    c->have_k = true;
    return AC_OK;
}

}  // extern "C"
