// cluster_kernels.cu -- k-means building blocks of the cluster-routed sparse
// layer (AdaCluster, arXiv 2604.18348, Sec. 3.1 and Sec. 3.2.2 Algorithm 1).
//
// Decisions (argmin labels, removal d_i < tau) are taken in fp32 with a fixed,
// sequential operation order and round-to-nearest intrinsics (no fused
// multiply-add), so labels, permutations and centres are reproducible
// bit-for-bit run to run.  Member sums are taken in ascending token order.
#include <cub/block/block_scan.cuh>

#include "ac_device.cuh"
#include "ac_internal.h"

namespace ac {

// ------------------------------------------------------------------ Sec. 3.1
// inv[i] = 1/||q_i||_2 (0 for a zero query), squares summed in dimension order.
__global__ void k_qnorm(const bf16 *__restrict__ Q, float *__restrict__ inv, int64_t rows, int d,
                        uint32_t *err) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(Q + i * d);
    float ss = 0.f;
    bool finite = true;
    for (int k8 = 0; k8 < d / 8; ++k8) {
        uint4 v = src[k8];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float a = __uint_as_float(w[t] << 16);
            float b = __uint_as_float(w[t] & 0xFFFF0000u);
            finite &= isfinite(a) && isfinite(b);
            ss = __fadd_rn(ss, __fmul_rn(a, a));
            ss = __fadd_rn(ss, __fmul_rn(b, b));
        }
    }
    if (!finite) set_err(err, DEV_ERR_NONFINITE);
    inv[i] = ss > 0.f ? __fdiv_rn(1.0f, __fsqrt_rn(ss)) : 0.f;
}

cudaError_t launch_qnorm(const bf16 *Q, float *inv, int64_t rows, int d, uint32_t *err, cudaStream_t s) {
    k_qnorm<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(Q, inv, rows, d, err);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// Load one row as fp32 (times inv when normalising).
template <int D, bool NORM>
__device__ __forceinline__ void load_row(const bf16 *__restrict__ src_row, float s, float (&x)[D]) {
    const uint4 *src = reinterpret_cast<const uint4 *>(src_row);
#pragma unroll
    for (int k8 = 0; k8 < D / 8; ++k8) {
        uint4 v = src[k8];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float a = __uint_as_float(w[t] << 16);
            float b = __uint_as_float(w[t] & 0xFFFF0000u);
            x[k8 * 8 + 2 * t] = NORM ? __fmul_rn(a, s) : a;
            x[k8 * 8 + 2 * t + 1] = NORM ? __fmul_rn(b, s) : b;
        }
    }
}

// ------------------------------------------------------------------ assignment
// One thread per row; centres staged through shared memory in chunks.
template <int D, bool NORM>
__global__ void __launch_bounds__(128) k_assign_exact(AssignArgs a) {
    constexpr int CH = 32;
    __shared__ __align__(16) float cs[CH * D];
    const int h = blockIdx.y;
    const int n = a.nrows ? a.nrows[h] : a.nrows_const;
    const int m = a.ncent ? a.ncent[h] : a.ncent_const;
    if ((int64_t)blockIdx.x * 128 >= n || m <= 0) return;
    const int r = blockIdx.x * 128 + threadIdx.x;
    const bool act = r < n;
    const float *Ch = a.C + (int64_t)h * a.cstride + (int64_t)(a.coff ? a.coff[h] : 0) * D;
    float x[D];
    if (act) {
        int64_t tok = a.rows ? a.rows[(int64_t)h * a.L + r] : r;
        float sc = NORM ? a.inv[(int64_t)h * a.L + tok] : 1.f;
        load_row<D, NORM>(a.X + ((int64_t)h * a.L + tok) * D, sc, x);
    } else {
#pragma unroll
        for (int k = 0; k < D; ++k) x[k] = 0.f;
    }
    float best = INFINITY;
    int arg = 0;
    for (int c0 = 0; c0 < m; c0 += CH) {
        const int nc = min(CH, m - c0);
        __syncthreads();
        for (int i = threadIdx.x; i < nc * D; i += 128) cs[i] = Ch[(int64_t)c0 * D + i];
        __syncthreads();
        for (int cc = 0; cc < nc; ++cc) {
            const float4 *c4 = reinterpret_cast<const float4 *>(cs + cc * D);
            float s = 0.f;
#pragma unroll
            for (int k4 = 0; k4 < D / 4; ++k4) {
                float4 cv = c4[k4];
                float t0 = __fsub_rn(x[4 * k4 + 0], cv.x);
                s = __fadd_rn(s, __fmul_rn(t0, t0));
                float t1 = __fsub_rn(x[4 * k4 + 1], cv.y);
                s = __fadd_rn(s, __fmul_rn(t1, t1));
                float t2 = __fsub_rn(x[4 * k4 + 2], cv.z);
                s = __fadd_rn(s, __fmul_rn(t2, t2));
                float t3 = __fsub_rn(x[4 * k4 + 3], cv.w);
                s = __fadd_rn(s, __fmul_rn(t3, t3));
            }
            if (s < best) {
                best = s;
                arg = c0 + cc;
            }
        }
    }
    if (act) {
        a.labels[(int64_t)h * a.L + r] = arg;
        if (a.dmin) a.dmin[(int64_t)h * a.L + r] = best;
    }
}

cudaError_t launch_assign_exact(const AssignArgs &a, cudaStream_t s) {
    int maxn = a.nrows ? (int)a.L : a.nrows_const;
    dim3 grid((unsigned)((maxn + 127) / 128), (unsigned)a.BH);
    if (grid.x == 0) return cudaSuccess;
    const bool norm = a.inv != nullptr;
    if (a.d == 128) {
        if (norm) k_assign_exact<128, true><<<grid, 128, 0, s>>>(a);
        else k_assign_exact<128, false><<<grid, 128, 0, s>>>(a);
    } else {
        if (norm) k_assign_exact<64, true><<<grid, 128, 0, s>>>(a);
        else k_assign_exact<64, false><<<grid, 128, 0, s>>>(a);
    }
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ stable sort
// One block (8 warps) per unit.  Warp w owns a contiguous chunk of the rows;
// per-warp histograms give each warp its first slot per label, then every
// warp scatters its chunk in order (warp-level match gives in-order ranks).
constexpr int SORT_WARPS = 8;
constexpr int SORT_SEGS = 16;                        // blocks per unit
constexpr int SORT_CHUNKS = SORT_SEGS * SORT_WARPS;  // contiguous row chunks per unit, one per warp

// Stable counting sort of the labels of every unit in three passes over
// SORT_CHUNKS contiguous row chunks (one warp each, SORT_SEGS blocks per unit):
// (1) per-chunk label histograms; (2) per unit, exclusive offsets of the labels
// and the first slot of every (label, chunk) in chunk order; (3) each chunk
// scatters its rows in order (warp-match ranks within 32 rows).  The result is
// the same as one sequential stable pass over the rows.
__global__ void __launch_bounds__(SORT_WARPS * 32) k_sort_hist(SortArgs a) {
    extern __shared__ int hist[];  // [SORT_WARPS][max_lab]
    const int seg = blockIdx.x, h = blockIdx.y;
    const int n = a.nrows ? a.nrows[h] : a.nrows_const;
    const int m = a.nlab ? a.nlab[h] : a.nlab_const;
    if (m <= 0) return;  // idle unit
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int *lab = a.labels + (int64_t)h * a.L;
    for (int i = tid; i < SORT_WARPS * m; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int ci = seg * SORT_WARPS + w;
    const int chunk = (n + SORT_CHUNKS - 1) / SORT_CHUNKS;
    const int beg = min(n, ci * chunk), end = min(n, beg + chunk);
    for (int i = beg + lane; i < end; i += 32) {
        const int l = lab[i];
        if ((unsigned)l < (unsigned)m) atomicAdd(&hist[w * m + l], 1);
    }
    __syncwarp();
    int *H = a.scratch + ((int64_t)h * SORT_CHUNKS + ci) * a.max_lab;
    for (int l = lane; l < m; l += 32) H[l] = hist[w * m + l];
}

__global__ void __launch_bounds__(256) k_sort_offsets(SortArgs a) {
    extern __shared__ int tot[];  // [max_lab]
    typedef cub::BlockScan<int, 256> Scan;
    __shared__ typename Scan::TempStorage scan_tmp;
    const int h = blockIdx.x, tid = threadIdx.x;
    const int n = a.nrows ? a.nrows[h] : a.nrows_const;
    const int m = a.nlab ? a.nlab[h] : a.nlab_const;
    if (m <= 0) return;
    int *H = a.scratch + (int64_t)h * SORT_CHUNKS * a.max_lab;
    for (int l = tid; l < m; l += 256) {
        int t = 0;
        for (int ci = 0; ci < SORT_CHUNKS; ++ci) t += H[(int64_t)ci * a.max_lab + l];
        tot[l] = t;
    }
    __syncthreads();
    const int sg = (m + 255) / 256;
    const int l0 = min(m, tid * sg), l1 = min(m, l0 + sg);
    int local = 0;
    for (int l = l0; l < l1; ++l) local += tot[l];
    int run;
    Scan(scan_tmp).ExclusiveSum(local, run);
    __syncthreads();
    for (int l = l0; l < l1; ++l) {
        const int t = tot[l];
        tot[l] = run;  // now the label's first slot
        run += t;
    }
    __syncthreads();
    int *offs = a.offs + (int64_t)h * a.offs_stride;
    for (int l = tid; l < m; l += 256) {
        int slot = tot[l];
        offs[l] = slot;
        const int first = slot;
        for (int ci = 0; ci < SORT_CHUNKS; ++ci) {
            const int c = H[(int64_t)ci * a.max_lab + l];
            H[(int64_t)ci * a.max_lab + l] = slot;  // first slot of chunk ci for label l
            slot += c;
        }
        if (a.counts) a.counts[(int64_t)h * a.counts_stride + l] = slot - first;
    }
    if (tid == 0) offs[m] = n;
}

__global__ void __launch_bounds__(SORT_WARPS * 32) k_sort_scatter(SortArgs a) {
    extern __shared__ int hist[];  // [SORT_WARPS][max_lab]
    const int seg = blockIdx.x, h = blockIdx.y;
    const int n = a.nrows ? a.nrows[h] : a.nrows_const;
    const int m = a.nlab ? a.nlab[h] : a.nlab_const;
    if (m <= 0) return;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int ci = seg * SORT_WARPS + w;
    const int chunk = (n + SORT_CHUNKS - 1) / SORT_CHUNKS;
    const int beg = min(n, ci * chunk), end = min(n, beg + chunk);
    if (beg >= end) return;  // no barrier below: warps leave independently
    const int *H = a.scratch + ((int64_t)h * SORT_CHUNKS + ci) * a.max_lab;
    int *hs = hist + w * m;
    for (int l = lane; l < m; l += 32) hs[l] = H[l];
    __syncwarp();
    const int *lab = a.labels + (int64_t)h * a.L;
    int *perm = a.perm + (int64_t)h * a.L;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = beg; base < end; base += 32) {
        const int i = base + lane;
        const bool v = i < end;
        int l = v ? lab[i] : -1 - lane;
        if (v && (unsigned)l >= (unsigned)m) l = -1 - lane;  // out of range: never placed
        const unsigned grp = __match_any_sync(0xFFFFFFFFu, l);
        const int rank = __popc(grp & lt);
        int slot = 0;
        if (l >= 0) slot = hs[l];
        __syncwarp();
        if (l >= 0) {
            perm[slot + rank] = i;
            if (rank == 0) hs[l] = slot + __popc(grp);
        }
        __syncwarp();
    }
}

// One block per unit (no scratch memory): per-warp histograms over contiguous
// chunks, offsets, then an in-order scatter.  Used when the caller provides
// no histogram scratch (the allocation-free entry point).
__global__ void __launch_bounds__(SORT_WARPS * 32) k_counting_sort(SortArgs a) {
    extern __shared__ int hist[];  // [SORT_WARPS][max_lab]
    typedef cub::BlockScan<int, SORT_WARPS * 32> Scan;
    __shared__ typename Scan::TempStorage scan_tmp;
    const int h = blockIdx.x;
    const int n = a.nrows ? a.nrows[h] : a.nrows_const;
    const int m = a.nlab ? a.nlab[h] : a.nlab_const;
    if (m <= 0) return;  // idle unit
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int *lab = a.labels + (int64_t)h * a.L;
    for (int i = tid; i < SORT_WARPS * m; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int chunk = (n + SORT_WARPS - 1) / SORT_WARPS;
    const int beg = min(n, w * chunk), end = min(n, beg + chunk);
    for (int i = beg + lane; i < end; i += 32) {
        int l = lab[i];
        if ((unsigned)l < (unsigned)m) atomicAdd(&hist[w * m + l], 1);
    }
    __syncthreads();
    const int seg = (m + blockDim.x - 1) / blockDim.x;
    const int l0 = min(m, tid * seg), l1 = min(m, l0 + seg);
    int local = 0;
    for (int l = l0; l < l1; ++l)
        for (int ww = 0; ww < SORT_WARPS; ++ww) local += hist[ww * m + l];
    int run;
    Scan(scan_tmp).ExclusiveSum(local, run);
    __syncthreads();
    int *offs = a.offs + (int64_t)h * a.offs_stride;
    for (int l = l0; l < l1; ++l) {
        offs[l] = run;
        int tot = 0;
        for (int ww = 0; ww < SORT_WARPS; ++ww) {
            int c = hist[ww * m + l];
            hist[ww * m + l] = run + tot;  // first slot of warp ww for label l
            tot += c;
        }
        if (a.counts) a.counts[(int64_t)h * a.counts_stride + l] = tot;
        run += tot;
    }
    if (tid == 0) offs[m] = n;
    __syncthreads();
    int *perm = a.perm + (int64_t)h * a.L;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = beg; base < end; base += 32) {
        const int i = base + lane;
        const bool v = i < end;
        int l = v ? lab[i] : -1 - lane;
        if (v && (unsigned)l >= (unsigned)m) l = -1 - lane;  // out of range: never placed
        const unsigned grp = __match_any_sync(0xFFFFFFFFu, l);
        const int rank = __popc(grp & lt);
        int slot = 0;
        if (l >= 0) slot = hist[w * m + l];
        __syncwarp();
        if (l >= 0) {
            perm[slot + rank] = i;
            if (rank == 0) hist[w * m + l] = slot + __popc(grp);
        }
        __syncwarp();
    }
}

cudaError_t launch_counting_sort(const SortArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)SORT_WARPS * a.max_lab * sizeof(int);
    cudaError_t e;
    if (!a.scratch) {
        if ((e = cudaFuncSetAttribute(k_counting_sort, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)(smem < 48 * 1024 ? 48 * 1024 : smem))) != cudaSuccess)
            return e;
        k_counting_sort<<<a.BH, SORT_WARPS * 32, smem, s>>>(a);
        AC_NOTE_LAUNCH();
        return cudaGetLastError();
    }
    if ((e = cudaFuncSetAttribute(k_sort_hist, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)(smem < 48 * 1024 ? 48 * 1024 : smem))) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(k_sort_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)(smem < 48 * 1024 ? 48 * 1024 : smem))) != cudaSuccess)
        return e;
    const dim3 grid(SORT_SEGS, a.BH);
    k_sort_hist<<<grid, SORT_WARPS * 32, smem, s>>>(a);
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_sort_offsets<<<a.BH, 256, (size_t)a.max_lab * sizeof(int), s>>>(a);
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_sort_scatter<<<grid, SORT_WARPS * 32, smem, s>>>(a);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ update
// One block per (cluster, unit), one thread per dimension; members summed in
// ascending order in fp32, then divided by the count.  The members' rows are
// scattered over the unit, so they are staged in shared memory by cp.async,
// UPD_BATCH rows per batch and UPD_STAGES batches in flight, while the
// threads add the rows of the oldest batch in order.
constexpr int UPD_BATCH = 32;
constexpr int UPD_STAGES = 4;

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <bool NORM>
__global__ void k_update(UpdateArgs a) {
    extern __shared__ __align__(16) uint8_t upd_sm[];
    bf16 *rows_s = reinterpret_cast<bf16 *>(upd_sm);                                    // [STAGES][BATCH][d]
    float *inv_s = reinterpret_cast<float *>(upd_sm + UPD_STAGES * UPD_BATCH * a.d * 2);  // [STAGES][BATCH]
    const int c = blockIdx.x, h = blockIdx.y, k = threadIdx.x;
    const int m = a.ncent ? a.ncent[h] : a.ncent_const;
    if (c >= m) return;
    const int *offs = a.offs + (int64_t)h * a.offs_stride;
    const int beg = offs[c], end = offs[c + 1];
    if (end <= beg) return;  // empty: keep the previous centre
    const int *perm = a.perm + (int64_t)h * a.L;
    const int *rows = a.rows ? a.rows + (int64_t)h * a.L : nullptr;
    const bf16 *X = a.X + (int64_t)h * a.L * a.d;
    const float *inv = NORM ? a.inv + (int64_t)h * a.L : nullptr;
    const int nthr = blockDim.x, pieces = a.d / 8;  // 16-byte pieces per row
    const int nb = (end - beg + UPD_BATCH - 1) / UPD_BATCH;
    // batch b: members beg + b*BATCH .. into stage b % STAGES
    auto issue = [&](int b) {
        if (b < nb) {
            const int st = b % UPD_STAGES;
            const int j0 = beg + b * UPD_BATCH;
            const int cnt = min(UPD_BATCH, end - j0);
            for (int q = k; q < cnt * pieces; q += nthr) {
                const int r = q / pieces, part = q % pieces;
                const int p = perm[j0 + r];
                const int t = rows ? rows[p] : p;
                cp_async16(rows_s + ((size_t)st * UPD_BATCH + r) * a.d + part * 8, X + (int64_t)t * a.d + part * 8);
            }
            if (NORM && k < cnt) {
                const int p = perm[j0 + k];
                inv_s[st * UPD_BATCH + k] = inv[rows ? rows[p] : p];
            }
        }
        cp_async_commit();  // an empty group past the last batch keeps the count uniform
    };
#pragma unroll 1
    for (int b = 0; b < UPD_STAGES - 1; ++b) issue(b);
    float s = 0.f;
#pragma unroll 1
    for (int b = 0; b < nb; ++b) {
        issue(b + UPD_STAGES - 1);
        cp_async_wait<UPD_STAGES - 1>();  // batch b has landed (this thread's copies)
        __syncthreads();                  // ... and every thread's
        const int st = b % UPD_STAGES;
        const int cnt = min(UPD_BATCH, end - beg - b * UPD_BATCH);
        if (k < a.d) {
            const bf16 *rs = rows_s + (size_t)st * UPD_BATCH * a.d + k;
            for (int r = 0; r < cnt; ++r) {
                float v = bf2f(rs[(size_t)r * a.d]);
                if (NORM) v = __fmul_rn(v, inv_s[st * UPD_BATCH + r]);
                s = __fadd_rn(s, v);
            }
        }
        __syncthreads();  // stage st is refilled by the next issue
    }
    cp_async_wait<0>();
    if (k < a.d) {
        const int off = a.coff ? a.coff[h] : 0;
        a.C[(int64_t)h * a.cstride + (int64_t)(off + c) * a.d + k] = __fdiv_rn(s, (float)(end - beg));
    }
}

// The same sums for small clusters (a few dozen members): each thread loads
// 32 members ahead from global memory, no staging.
template <bool NORM>
__global__ void k_update_direct(UpdateArgs a) {
    const int c = blockIdx.x, h = blockIdx.y, k = threadIdx.x;
    const int m = a.ncent ? a.ncent[h] : a.ncent_const;
    if (c >= m || k >= a.d) return;
    const int *offs = a.offs + (int64_t)h * a.offs_stride;
    const int beg = offs[c], end = offs[c + 1];
    if (end <= beg) return;  // empty: keep the previous centre
    const int *perm = a.perm + (int64_t)h * a.L;
    const int *rows = a.rows ? a.rows + (int64_t)h * a.L : nullptr;
    const bf16 *X = a.X + (int64_t)h * a.L * a.d;
    const float *inv = NORM ? a.inv + (int64_t)h * a.L : nullptr;
    float s = 0.f;
    constexpr int U = 32;
    int j = beg;
    for (; j + U <= end; j += U) {
        int tok[U];
        float v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) tok[u] = perm[j + u];
        if (rows) {
#pragma unroll
            for (int u = 0; u < U; ++u) tok[u] = rows[tok[u]];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            v[u] = bf2f(X[(int64_t)tok[u] * a.d + k]);
            if (NORM) v[u] = __fmul_rn(v[u], inv[tok[u]]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) s = __fadd_rn(s, v[u]);
    }
    for (; j < end; ++j) {
        const int p = perm[j];
        const int t = rows ? rows[p] : p;
        float v = bf2f(X[(int64_t)t * a.d + k]);
        if (NORM) v = __fmul_rn(v, inv[t]);
        s = __fadd_rn(s, v);
    }
    const int off = a.coff ? a.coff[h] : 0;
    a.C[(int64_t)h * a.cstride + (int64_t)(off + c) * a.d + k] = __fdiv_rn(s, (float)(end - beg));
}

cudaError_t launch_update(const UpdateArgs &a, cudaStream_t s) {
    dim3 grid((unsigned)a.max_cent, (unsigned)a.BH);
    // few, large clusters (queries): staged batches; many small ones: direct
    if ((int64_t)a.max_cent * 256 <= a.L) {
        const size_t smem = (size_t)UPD_STAGES * UPD_BATCH * (a.d * 2 + 4);
        if (a.inv) k_update<true><<<grid, a.d, smem, s>>>(a);
        else k_update<false><<<grid, a.d, smem, s>>>(a);
    } else {
        if (a.inv) k_update_direct<true><<<grid, a.d, 0, s>>>(a);
        else k_update_direct<false><<<grid, a.d, 0, s>>>(a);
    }
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ seeding
__global__ void k_seed(SeedArgs a) {
    const int h = blockIdx.y;
    const int j = blockIdx.x * blockDim.y + threadIdx.y;
    const int m = a.m ? a.m[h] : a.m_const;
    if (j >= m) return;
    const int64_t n = a.nrows ? a.nrows[h] : a.nrows_const;
    const int64_t pos = stratum_pick(a.seed, h, a.tag, n, m, j);
    const int64_t tok = a.rows ? a.rows[(int64_t)h * a.L + pos] : pos;
    const float sc = a.inv ? a.inv[(int64_t)h * a.L + tok] : 1.f;
    const int off = a.coff ? a.coff[h] : 0;
    float *dst = a.C + (int64_t)h * a.cstride + (int64_t)(off + j) * a.d;
    const bf16 *src = a.X + ((int64_t)h * a.L + tok) * a.d;
    for (int k = threadIdx.x; k < a.d; k += blockDim.x) {
        float v = bf2f(src[k]);
        dst[k] = a.inv ? __fmul_rn(v, sc) : v;
    }
}

cudaError_t launch_seed(const SeedArgs &a, cudaStream_t s) {
    dim3 block(32, 8);
    dim3 grid((unsigned)((a.max_m + 7) / 8), (unsigned)a.BH);
    if (grid.x == 0) return cudaSuccess;
    k_seed<<<grid, block, 0, s>>>(a);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ Algorithm 1 helpers
__global__ void k_iota_rows(int *u_idx, int *u_cnt, int L) {
    const int h = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < L) u_idx[(int64_t)h * L + i] = i;
    if (i == 0) u_cnt[h] = L;
}

cudaError_t launch_iota_rows(int *u_idx, int *u_cnt, int BH, int L, cudaStream_t s) {
    k_iota_rows<<<dim3((L + 255) / 256, BH), 256, 0, s>>>(u_idx, u_cnt, L);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// d_i = sqrt of the winning squared distance; stage 0 also accumulates the
// exact fixed-point sum floor(d_i * 2^24) used by the mean rule for tau.
__global__ void k_stage_dist(const float *__restrict__ dmin, float *__restrict__ dist,
                             const int *__restrict__ u_cnt, const int *__restrict__ st_m, int64_t L,
                             unsigned long long *tau_acc) {
    const int h = blockIdx.y;
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    const bool act = st_m[h] > 0 && i < u_cnt[h];
    unsigned long long q = 0;
    if (act) {
        float dd = __fsqrt_rn(dmin[(int64_t)h * L + i]);
        dist[(int64_t)h * L + i] = dd;
        q = __double2ull_rz(__dmul_rn((double)dd, 16777216.0));
    }
    if (tau_acc) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) q += __shfl_down_sync(0xFFFFFFFFu, q, o);
        if ((threadIdx.x & 31) == 0 && q) atomicAdd(tau_acc, q);
    }
}

cudaError_t launch_stage_dist(const float *dmin, float *dist, const int *u_cnt, const int *st_m,
                              int64_t L, int BH, unsigned long long *tau_acc, cudaStream_t s) {
    k_stage_dist<<<dim3((unsigned)((L + 255) / 256), BH), 256, 0, s>>>(dmin, dist, u_cnt, st_m, L, tau_acc);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// tau = factor * mean, the mean formed from the fixed-point sum in fp64.
__global__ void k_tau_mean(const unsigned long long *acc, int64_t n, float factor, float *tau) {
    double mean = __ddiv_rn(__ddiv_rn(__ull2double_rn(*acc), 16777216.0), (double)n);
    *tau = __double2float_rn(__dmul_rn((double)factor, mean));
}

cudaError_t launch_tau_mean(const unsigned long long *tau_acc, const int *, int64_t n_total, float factor,
                            float *tau, cudaStream_t s) {
    k_tau_mean<<<1, 1, 0, s>>>(tau_acc, n_total, factor, tau);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// Nearest-rank percentile of the pooled stage-0 distances by a 4-pass
// most-significant-digit radix select on the bit patterns (d_i >= 0, so the
// unsigned order of the bits is the numeric order).
// radix[0..255]: histogram; radix[256]: prefix; radix[257]: mask; radix[258]: rank.
__global__ void k_radix_hist(const float *__restrict__ dist, const int *__restrict__ st_m, int64_t L,
                             uint32_t *radix, int shift) {
    __shared__ uint32_t hs[256];
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hs[i] = 0;
    __syncthreads();
    const int h = blockIdx.y;
    const uint32_t prefix = radix[256], mask = radix[257];
    if (st_m[h] > 0) {
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L;
             i += (int64_t)gridDim.x * blockDim.x) {
            uint32_t b = __float_as_uint(dist[(int64_t)h * L + i]);
            if ((b & mask) == prefix) atomicAdd(&hs[(b >> shift) & 255u], 1u);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (hs[i]) atomicAdd(&radix[i], hs[i]);
}

__global__ void k_radix_pick(uint32_t *radix, int shift, float *tau, int last) {
    if (threadIdx.x != 0) return;
    uint32_t rank = radix[258], cum = 0;
    int dg = 255;
    for (int i = 0; i < 256; ++i) {
        if (cum + radix[i] > rank) {
            dg = i;
            break;
        }
        cum += radix[i];
    }
    radix[258] = rank - cum;
    radix[256] |= (uint32_t)dg << shift;
    radix[257] |= 255u << shift;
    for (int i = 0; i < 256; ++i) radix[i] = 0;
    if (last) *tau = __uint_as_float(radix[256]);
}

__global__ void k_radix_init(uint32_t *radix, uint32_t rank) {
    for (int i = threadIdx.x; i < 259; i += blockDim.x) radix[i] = (i == 258) ? rank : 0u;
}

cudaError_t launch_tau_percentile(const float *dist, const int *st_m, int64_t L, int BH, int64_t n_total,
                                  int permille, uint32_t *radix, float *tau, cudaStream_t s) {
    int64_t idx = ((int64_t)permille * n_total + 999) / 1000 - 1;
    if (idx < 0) idx = 0;
    if (idx > n_total - 1) idx = n_total - 1;
    k_radix_init<<<1, 256, 0, s>>>(radix, (uint32_t)idx);
    AC_NOTE_LAUNCH();
    for (int p = 0; p < 4; ++p) {
        int shift = 24 - 8 * p;
        k_radix_hist<<<dim3(64, BH), 256, 0, s>>>(dist, st_m, L, radix, shift);
        AC_NOTE_LAUNCH();
        k_radix_pick<<<1, 32, 0, s>>>(radix, shift, tau, p == 3);
        AC_NOTE_LAUNCH();
    }
    return cudaGetLastError();
}

// Algorithm 1 lines 13-18: keep the members of U with d_i >= tau (in order),
// record the stage of the others.  One block per unit; order-preserving scan.
__global__ void __launch_bounds__(1024) k_remove(const float *__restrict__ dist, const float *__restrict__ tau,
                                                 const int *__restrict__ u_idx, int *__restrict__ u_idx2,
                                                 int *__restrict__ u_cnt, const int *__restrict__ st_m,
                                                 int *__restrict__ removed_stage, int stage, int64_t L) {
    typedef cub::BlockScan<int, 1024> Scan;
    __shared__ typename Scan::TempStorage tmp;
    __shared__ int base_s;
    const int h = blockIdx.x;
    if (st_m[h] <= 0) return;
    const int n = u_cnt[h];
    const float t = *tau;
    if (threadIdx.x == 0) base_s = 0;
    __syncthreads();
    for (int c0 = 0; c0 < n; c0 += 1024) {
        const int i = c0 + threadIdx.x;
        int keep = 0, tok = 0;
        if (i < n) {
            tok = u_idx[(int64_t)h * L + i];
            float dd = dist[(int64_t)h * L + i];
            if (dd < t) removed_stage[(int64_t)h * L + tok] = stage;
            else keep = 1;
        }
        int pos, tot;
        Scan(tmp).ExclusiveSum(keep, pos, tot);
        const int base = base_s;
        if (keep) u_idx2[(int64_t)h * L + base + pos] = tok;
        __syncthreads();
        if (threadIdx.x == 0) base_s = base + tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) u_cnt[h] = base_s;
}

cudaError_t launch_remove(const float *dist, const float *tau, int *u_idx, int *u_idx2, int *u_cnt,
                          const int *st_m, int *removed_stage, int stage, int64_t L, int BH, cudaStream_t s) {
    k_remove<<<BH, 1024, 0, s>>>(dist, tau, u_idx, u_idx2, u_cnt, st_m, removed_stage, stage, L);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ Sec. 3.2.1 stats
// One block per (cluster, unit), one thread per dimension: count, exact
// per-dimension max/min, and (thread 0) SSE over members in ascending order.
__global__ void k_key_stats(StatsArgs a) {
    const int c = blockIdx.x, h = blockIdx.y, k = threadIdx.x;
    const int nk = a.n_k[h];
    const int64_t ci = (int64_t)h * a.Ccap + c;
    if (c >= nk) {
        if (k == 0) {
            a.counts[ci] = 0;
            a.sse[ci] = 0.f;
        }
        a.kmax[ci * a.d + k] = __float2bfloat16(0.f);
        a.kmin[ci * a.d + k] = __float2bfloat16(0.f);
        return;
    }
    const int *offs = a.offs + (int64_t)h * a.offs_stride;
    const int beg = offs[c], end = offs[c + 1];
    const int *perm = a.perm + (int64_t)h * a.L;
    const bf16 *K = a.K + (int64_t)h * a.L * a.d;
    // 16 members in flight per step (scattered rows); max and min are exact
    // in any order, the SSE is summed in member order
    constexpr int U = 16;
    float mx = 0.f, mn = 0.f;  // an empty cluster keeps 0 (and count 0)
    if (end > beg) mx = mn = bf2f(K[(int64_t)perm[beg] * a.d + k]);
    int j = beg + 1;
    for (; j + U <= end; j += U) {
        float v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) v[u] = bf2f(K[(int64_t)perm[j + u] * a.d + k]);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            mx = v[u] > mx ? v[u] : mx;
            mn = v[u] < mn ? v[u] : mn;
        }
    }
    for (; j < end; ++j) {
        const float v = bf2f(K[(int64_t)perm[j] * a.d + k]);
        mx = v > mx ? v : mx;
        mn = v < mn ? v : mn;
    }
    a.kmax[ci * a.d + k] = __float2bfloat16(mx);
    a.kmin[ci * a.d + k] = __float2bfloat16(mn);
    if (k == 0) {
        float se = 0.f;
        const float *dm = a.dmin + (int64_t)h * a.L;
        int i = beg;
        for (; i + U <= end; i += U) {
            float v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) v[u] = dm[perm[i + u]];
#pragma unroll
            for (int u = 0; u < U; ++u) se = __fadd_rn(se, v[u]);
        }
        for (; i < end; ++i) se = __fadd_rn(se, dm[perm[i]]);
        a.sse[ci] = se;
        a.counts[ci] = end - beg;
    }
}

// MSE = (sum of the cluster SSEs in cluster order) / L and Comp = 1/MSE.
__global__ void k_head_comp(StatsArgs a) {
    const int h = blockIdx.x * blockDim.x + threadIdx.x;
    if (h >= a.BH) return;
    float tot = 0.f;
    for (int c = 0; c < a.n_k[h]; ++c) tot = __fadd_rn(tot, a.sse[(int64_t)h * a.Ccap + c]);
    float mse = __fdiv_rn(tot, (float)a.L);
    a.mse[h] = mse;
    a.comp[h] = __fdiv_rn(1.0f, mse);
}

cudaError_t launch_key_stats(const StatsArgs &a, cudaStream_t s) {
    k_key_stats<<<dim3(a.Ccap, a.BH), a.d, 0, s>>>(a);
    AC_NOTE_LAUNCH();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_head_comp<<<(a.BH + 127) / 128, 128, 0, s>>>(a);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ gathers
// Xp[h, pos] = X[h, perm[h, pos]]: 16-byte lanes, one row per d/8 lanes.
__global__ void k_permute_rows(const bf16 *__restrict__ X, const int *__restrict__ perm,
                               bf16 *__restrict__ Xp, int64_t L, int d, int64_t total_rows) {
    const int lanes_per_row = d / 8;
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = g / lanes_per_row;
    const int part = (int)(g % lanes_per_row);
    if (row >= total_rows) return;
    const int64_t h = row / L;
    const int64_t src = h * L + perm[row];
    reinterpret_cast<uint4 *>(Xp + row * d)[part] = reinterpret_cast<const uint4 *>(X + src * d)[part];
}

cudaError_t launch_permute_rows(const bf16 *X, const int *perm, bf16 *Xp, int64_t L, int d, int BH,
                                cudaStream_t s) {
    const int64_t rows = (int64_t)BH * L;
    const int64_t threads = rows * (d / 8);
    k_permute_rows<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(X, perm, Xp, L, d, rows);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// Kp[h, 8 pgoff[h, c] + i] = K[h, perm[h, offs[h, c] + i]] (and V alike): the
// keys of cluster c in order, the cluster starting on an 8-row group.
__global__ void k_permute_kv_padded(const bf16 *__restrict__ K, const bf16 *__restrict__ V,
                                    const int *__restrict__ perm, const int *__restrict__ labels,
                                    const int *__restrict__ offs, int offs_stride, const int *__restrict__ pgoff,
                                    int Ccap, bf16 *__restrict__ Kp, bf16 *__restrict__ Vp, int64_t L, int64_t Lpad,
                                    int d, int64_t total_rows) {
    const int lanes_per_row = d / 8;
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t row = g / lanes_per_row;
    const int part = (int)(g % lanes_per_row);
    if (row >= total_rows) return;
    const int64_t h = row / L, pos = row % L;
    const int tok = perm[row];
    const int c = labels[h * L + tok];
    const int64_t dst = h * Lpad + 8ll * pgoff[h * Ccap + c] + (pos - offs[h * offs_stride + c]);
    const int64_t src = h * L + tok;
    reinterpret_cast<uint4 *>(Kp + dst * d)[part] = reinterpret_cast<const uint4 *>(K + src * d)[part];
    reinterpret_cast<uint4 *>(Vp + dst * d)[part] = reinterpret_cast<const uint4 *>(V + src * d)[part];
}

cudaError_t launch_permute_kv_padded(const bf16 *K, const bf16 *V, const int *perm, const int *labels,
                                     const int *offs, int offs_stride, const int *pgoff, int Ccap, bf16 *Kp,
                                     bf16 *Vp, int64_t L, int64_t Lpad, int d, int BH, cudaStream_t s) {
    const int64_t rows = (int64_t)BH * L;
    const int64_t threads = rows * (d / 8);
    k_permute_kv_padded<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(K, V, perm, labels, offs, offs_stride,
                                                                          pgoff, Ccap, Kp, Vp, L, Lpad, d, rows);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

}  // namespace ac
