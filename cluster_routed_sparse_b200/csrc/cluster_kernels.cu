// cluster_kernels.cu -- k-means building blocks of the cluster-routed sparse
// layer (AdaCluster, arXiv 2604.18348, Sec. 3.1 and Sec. 3.2.2 Algorithm 1).
//
// Decisions (argmin labels, removal d_i < tau) are taken in fp32 with a fixed,
// sequential operation order and round-to-nearest intrinsics (no fused
// multiply-add), so labels, permutations and centres are reproducible
// bit-for-bit run to run.  Member sums are taken in ascending token order.
#include <cub/block/block_reduce.cuh>
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

// Pass (2) in two kernels over (unit, block of 32 labels), so that every SM
// takes part: the lanes of a warp read 32 consecutive labels of one chunk row
// (coalesced), the 8 warps of a block 16 chunks each.
//  k_sort_totals:  tot[h, l] = sum over the chunks of the count of label l;
//  k_sort_offsets: offs[h, l] = sum of tot[h, l'] for l' < l, counts[h, l] = tot,
//                  and every (label, chunk) histogram entry replaced by the first
//                  slot of that chunk's rows of the label.
constexpr int SORT_LB = 32;                        // labels per block
constexpr int SORT_CPW = SORT_CHUNKS / SORT_WARPS;  // chunks per warp

__global__ void __launch_bounds__(SORT_WARPS * 32) k_sort_totals(SortArgs a, int *tot) {
    __shared__ int part[SORT_WARPS][SORT_LB];
    const int h = blockIdx.y, l = blockIdx.x * SORT_LB + (threadIdx.x & 31), w = threadIdx.x >> 5;
    const int m = a.nlab ? a.nlab[h] : a.nlab_const;
    if (m <= 0 || blockIdx.x * SORT_LB >= m) return;
    const int *H = a.scratch + (int64_t)h * SORT_CHUNKS * a.max_lab;
    int t = 0;
    if (l < m) {
#pragma unroll
        for (int c = 0; c < SORT_CPW; ++c) t += H[(int64_t)(w * SORT_CPW + c) * a.max_lab + l];
    }
    part[w][threadIdx.x & 31] = t;
    __syncthreads();
    if (w == 0 && l < m) {
        int s = 0;
#pragma unroll
        for (int i = 0; i < SORT_WARPS; ++i) s += part[i][threadIdx.x];
        tot[(int64_t)h * a.max_lab + l] = s;
    }
}

__global__ void __launch_bounds__(SORT_WARPS * 32) k_sort_offsets(SortArgs a, const int *tot) {
    typedef cub::BlockReduce<int, SORT_WARPS * 32> Red;
    __shared__ typename Red::TempStorage red_tmp;
    __shared__ int base_s, lab_off[SORT_LB];
    __shared__ int part[SORT_WARPS][SORT_LB];
    const int h = blockIdx.y, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int l0 = blockIdx.x * SORT_LB, l = l0 + lane;
    const int n = a.nrows ? a.nrows[h] : a.nrows_const;
    const int m = a.nlab ? a.nlab[h] : a.nlab_const;
    if (m <= 0 || l0 >= m) return;
    const int *T = tot + (int64_t)h * a.max_lab;
    // rows of every label before this block's
    int before = 0;
    for (int i = threadIdx.x; i < l0; i += SORT_WARPS * 32) before += T[i];
    before = Red(red_tmp).Sum(before);
    if (threadIdx.x == 0) base_s = before;
    __syncthreads();
    if (w == 0) {
        const int t = l < m ? T[l] : 0;
        int incl = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        lab_off[lane] = base_s + incl - t;
        if (l < m) {
            a.offs[(int64_t)h * a.offs_stride + l] = base_s + incl - t;
            if (a.counts) a.counts[(int64_t)h * a.counts_stride + l] = t;
        }
        if (l0 + SORT_LB >= m && lane == 0) a.offs[(int64_t)h * a.offs_stride + m] = n;
    }
    // this warp's chunks of label l: their counts, the warp's share, then first slots
    int *H = a.scratch + (int64_t)h * SORT_CHUNKS * a.max_lab;
    int cv[SORT_CPW], mine = 0;
#pragma unroll
    for (int c = 0; c < SORT_CPW; ++c) {
        cv[c] = l < m ? H[(int64_t)(w * SORT_CPW + c) * a.max_lab + l] : 0;
        mine += cv[c];
    }
    part[w][lane] = mine;
    __syncthreads();
    int slot = lab_off[lane];
    for (int i = 0; i < w; ++i) slot += part[i][lane];
    if (l < m) {
#pragma unroll
        for (int c = 0; c < SORT_CPW; ++c) {
            H[(int64_t)(w * SORT_CPW + c) * a.max_lab + l] = slot;  // first slot of this chunk's rows of label l
            slot += cv[c];
        }
    }
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
    {
        // the per-label totals follow the chunk histograms of all units in the scratch
        int *tot = a.scratch + (int64_t)a.BH * SORT_CHUNKS * a.max_lab;
        const dim3 g((unsigned)((a.max_lab + SORT_LB - 1) / SORT_LB), (unsigned)a.BH);
        k_sort_totals<<<g, SORT_WARPS * 32, 0, s>>>(a, tot);
        AC_NOTE_LAUNCH();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        k_sort_offsets<<<g, SORT_WARPS * 32, 0, s>>>(a, tot);
        AC_NOTE_LAUNCH();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    k_sort_scatter<<<grid, SORT_WARPS * 32, smem, s>>>(a);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ member streaming
// The centre update and the key statistics both walk the members of every
// cluster in ascending member order.  Members are scattered over the unit, so
// a producer warp gathers their rows (16-byte cp.async pieces, completion on
// an mbarrier) into a ring of MS_STAGES shared-memory stages of BATCH rows,
// and d consumer threads (one per dimension) reduce the stages in order.
// The grid is persistent: block g takes a contiguous range of the flat
// (unit, cluster) list holding about 1/G of the work (members plus MS_W per
// cluster for its partly filled last batch), so the member indices it reads
// (perm) are contiguous too; the producer fetches them in windows of MS_WIN,
// three windows ahead.
constexpr int MS_STAGES = 4;
constexpr int MS_WIN = 256;   // member indices per window
constexpr int MS_WSLOTS = 4;  // window ring
constexpr int MS_W = 16;      // work of one cluster beyond its members, in rows
enum { MS_FIRST = 1, MS_LAST = 2, MS_EMPTY = 4, MS_END = 8 };
enum { MS_UPDATE = 0, MS_UPDATE_NORM = 1, MS_STATS = 2 };

struct MsArgs {
    const bf16 *X; const float *inv; int64_t L;
    const int *rows;                    // [BH, L] or null (update only)
    const int *perm; const int *offs; int offs_stride;
    const int *ncent; int ncent_const;  // clusters c < m(h) hold members
    int maxc, BH;                       // flat list: f = h * maxc + c
    float *C; int64_t cstride; const int *coff;  // update: centres written; stats: centres read
    float *dmin; float *dsorted; bf16 *kmax; bf16 *kmin;  // stats
    uint32_t *err;
};

template <int D, int MODE>
struct MsLayout {
    // the query update takes 64-row stages: its clusters are few and large
    static constexpr int BATCH = MODE == MS_UPDATE_NORM ? 64 : 32;
    // stats rows are padded: per-row 16-byte reads then hit distinct banks
    static constexpr uint32_t ROWB = MODE == MS_STATS ? D * 2 + 16 : D * 2;
    static constexpr uint32_t STAGE = BATCH * ROWB;
    static constexpr uint32_t OFF_AUX = MS_STAGES * STAGE;                   // [STAGES][BATCH] inv or token
    static constexpr uint32_t OFF_META = OFF_AUX + MS_STAGES * BATCH * 4;   // [STAGES] int4
    static constexpr uint32_t OFF_BAR = OFF_META + MS_STAGES * 16;          // full[STAGES], empty[STAGES]
    static constexpr uint32_t OFF_CENT = OFF_BAR + 2 * MS_STAGES * 8;       // [STAGES][D] fp32 centre (stats)
    static constexpr uint32_t OFF_WDESC = OFF_CENT + (MODE == MS_STATS ? MS_STAGES * D * 4 : 0);
    static constexpr uint32_t OFF_WIN = OFF_WDESC + MS_WSLOTS * 16;         // [WSLOTS][WIN] int (producer)
    static constexpr uint32_t BYTES = OFF_WIN + MS_WSLOTS * MS_WIN * 4;
};

// Work position of flat cluster f: h S + (start of cluster c + MS_W c) with
// S = L + MS_W maxc, or (h + 1) S for a slot c >= m(h).  Non-decreasing in f.
__device__ __forceinline__ int64_t ms_key(const MsArgs &a, int f) {
    const int h = f / a.maxc, c = f - h * a.maxc;
    const int m = a.ncent ? a.ncent[h] : a.ncent_const;
    const int64_t S = a.L + (int64_t)MS_W * a.maxc;
    return (int64_t)h * S + (c < m ? a.offs[(int64_t)h * a.offs_stride + c] + (int64_t)MS_W * c : S);
}

// Block g's range [fs, fe): fs(g) = the first f whose key reaches g M / G
// (M = BH S), found by a 16-ary search per half warp (lanes 0-15: g,
// lanes 16-31: g + 1).  Every cluster lands in exactly one range.
__device__ __forceinline__ void ms_range(const MsArgs &a, int total, int G, int lane, int &fs, int &fe) {
    const int half = lane >> 4, hl = lane & 15;
    const int g = (int)blockIdx.x + half;
    const int64_t S = a.L + (int64_t)MS_W * a.maxc;
    const int64_t T = (int64_t)a.BH * S * g / G;
    int lo = total, hi = total;  // the answer lies in [lo, hi]
    if (g < G) {
        const int64_t h0 = min(T / S, (int64_t)a.BH - 1);
        lo = (int)max((int64_t)0, (h0 - 1) * a.maxc);
        hi = (int)min((int64_t)total, (h0 + 1) * a.maxc);
    }
    while (__any_sync(0xFFFFFFFFu, hi > lo)) {
        const int step = hi > lo ? (hi - lo + 15) / 16 : 1;
        const int fp = lo + hl * step;
        const bool ge = hi <= lo || fp >= hi || ms_key(a, fp) >= T;
        const unsigned b = (__ballot_sync(0xFFFFFFFFu, ge) >> (16 * half)) & 0xFFFFu;
        if (hi > lo) {
            if (b == 0u) {
                lo = lo + 15 * step + 1;
            } else {
                const int first = __ffs(b) - 1;
                if (first == 0) {
                    hi = lo;
                } else {
                    hi = lo + first * step;
                    lo = lo + (first - 1) * step + 1;
                }
            }
        }
    }
    fs = __shfl_sync(0xFFFFFFFFu, lo, 0);
    fe = __shfl_sync(0xFFFFFFFFu, lo, 16);
}

// The producer's queue of upcoming clusters: lane l examines cluster fbase + l
// (one latency for 32 clusters).  An item is a cluster with members; the
// statistics also emit the empty clusters c < m(h) (as MS_EMPTY items; the
// slots c >= m(h) are zeroed apart), the update skips them (they keep their
// centre).
struct MsQueue {
    int f, beg, end;  // this lane's cluster
    unsigned mask;    // lanes still holding an item
    int fbase, fend;
};

template <int MODE>
__device__ __forceinline__ void ms_refill(const MsArgs &a, int lane, MsQueue &q) {
    const int fl = q.fbase + lane;
    bool v = false;
    int b = 0, e = 0;
    if (fl < q.fend) {
        const int h = fl / a.maxc, c = fl - h * a.maxc;
        const int m = a.ncent ? a.ncent[h] : a.ncent_const;
        if (c < m) {
            const int *o = a.offs + (int64_t)h * a.offs_stride + c;
            b = o[0];
            e = o[1];
            v = e > b || MODE == MS_STATS;
        }
    }
    q.f = fl;
    q.beg = b;
    q.end = e;
    q.mask = __ballot_sync(0xFFFFFFFFu, v);
    q.fbase += 32;
}

template <int MODE>
__device__ __forceinline__ bool ms_pop(const MsArgs &a, int lane, MsQueue &q, int &f, int &beg, int &end) {
    while (q.mask == 0u && q.fbase < q.fend) ms_refill<MODE>(a, lane, q);
    if (q.mask == 0u) return false;
    const int src = __ffs(q.mask) - 1;
    q.mask &= q.mask - 1u;
    f = __shfl_sync(0xFFFFFFFFu, q.f, src);
    beg = __shfl_sync(0xFFFFFFFFu, q.beg, src);
    end = __shfl_sync(0xFFFFFFFFu, q.end, src);
    return true;
}

__device__ __forceinline__ void ms_cp16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void ms_cp4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void ms_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void ms_wait2() { asm volatile("cp.async.wait_group 2;" ::: "memory"); }
// Arrives on bar once every cp.async this thread issued so far has landed
// (counted in the barrier's expected arrivals).
__device__ __forceinline__ void ms_cp_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Exact squared distance of a bf16 row (in shared memory) to an fp32 centre
// (in shared memory): per dimension the difference and its square are
// rounded to fp32, then added over the dimensions in order.
template <int D>
__device__ __forceinline__ float ms_sqdist(const uint8_t *row, const float *cent) {
    const uint4 *xr = reinterpret_cast<const uint4 *>(row);
    const float4 *c4 = reinterpret_cast<const float4 *>(cent);
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < D / 8; ++q) {
        const uint4 xv = xr[q];
        const float4 ca = c4[2 * q], cb = c4[2 * q + 1];
        const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
        const float cc[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
            const uint64_t x2 = f2_pack(__uint_as_float(w[pr] << 16), __uint_as_float(w[pr] & 0xFFFF0000u));
            const uint64_t d2 = f2_sub(x2, f2_pack(cc[2 * pr], cc[2 * pr + 1]));
            float s0, s1;
            f2_unpack(f2_mul(d2, d2), s0, s1);
            acc = __fadd_rn(acc, s0);
            acc = __fadd_rn(acc, s1);
        }
    }
    return acc;
}

template <int D, int MODE>
__global__ void __launch_bounds__(D + 32) k_member_stream(MsArgs a) {
    using LY = MsLayout<D, MODE>;
    constexpr int BATCH = LY::BATCH;
    extern __shared__ __align__(128) uint8_t ms_sm[];
    const uint32_t sbase = smem_u32(ms_sm);
    const uint32_t bar_full = sbase + LY::OFF_BAR, bar_empty = bar_full + MS_STAGES * 8;
    int4 *meta = reinterpret_cast<int4 *>(ms_sm + LY::OFF_META);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NCW = D / 32;  // consumer warps
    if (tid == 0) {
        for (int i = 0; i < MS_STAGES; ++i) {
            mbar_init(bar_full + 8 * i, 33);  // 32 cp.async arrivals + lane 0's
            mbar_init(bar_empty + 8 * i, NCW);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const int total = a.BH * a.maxc, G = gridDim.x;
    if (MODE == MS_STATS && warp < NCW) {
        // slots without a cluster (c >= m(h)): bounds 0
        for (int f = blockIdx.x; f < total; f += G) {
            const int h = f / a.maxc, c = f - h * a.maxc;
            if (c < a.ncent[h]) continue;
            a.kmax[(int64_t)f * D + tid] = __float2bfloat16(0.f);
            a.kmin[(int64_t)f * D + tid] = __float2bfloat16(0.f);
        }
    }
    if (warp == NCW) {
        // ---------------- producer warp: 16-byte pieces, PPR lanes per row,
        // RPI rows per instruction
        constexpr int PPR = D / 8, RPI = 32 / PPR;
        int4 *wdesc = reinterpret_cast<int4 *>(ms_sm + LY::OFF_WDESC);
        const int *win = reinterpret_cast<const int *>(ms_sm + LY::OFF_WIN);
        const uint32_t win_s = sbase + LY::OFF_WIN;
        MsQueue q{0, 0, 0, 0u, 0, 0};
        ms_range(a, total, G, lane, q.fbase, q.fend);
        // window frontier: (f, beg, end) and the window start ws
        int ff = 0, fbeg = 0, fend = 0, ws = 0;
        bool fhave = ms_pop<MODE>(a, lane, q, ff, fbeg, fend);
        ws = fbeg;
        // window n -> slot n % WSLOTS: descriptor and member indices, one commit group
        auto issue_window = [&](uint32_t n) {
            const uint32_t sl = n % MS_WSLOTS;
            if (lane == 0) wdesc[sl] = fhave ? make_int4(ff, fbeg, fend, ws) : make_int4(-1, 0, 0, 0);
            if (fhave) {
                const int *src = a.perm + (int64_t)(ff / a.maxc) * a.L;
#pragma unroll
                for (int i = 0; i < MS_WIN / 32; ++i) {
                    const int pos = ws + 32 * i + lane;
                    if (pos < fend) ms_cp4(win_s + (sl * MS_WIN + 32 * i + lane) * 4, src + pos);
                }
                // advance the frontier
                if (ws + MS_WIN < fend) {
                    ws += MS_WIN;
                } else {
                    fhave = ms_pop<MODE>(a, lane, q, ff, fbeg, fend);
                    ws = fbeg;
                }
            }
            ms_commit();
        };
        issue_window(0);
        issue_window(1);
        issue_window(2);
        uint32_t it = 0;
        bool ok = true;
        for (uint32_t w = 0; ok; ++w) {
            issue_window(w + 3);
            ms_wait2();  // window w has landed (each lane reads the entries it loaded)
            __syncwarp();
            const int4 dw = wdesc[w % MS_WSLOTS];
            if (dw.x < 0) break;
            const int hh = dw.x / a.maxc;
            const int *wc = win + (w % MS_WSLOTS) * MS_WIN;
            const bf16 *src = a.X + (int64_t)hh * a.L * D + (lane % PPR) * 8;
            for (int i = 0; i < MS_WIN / BATCH; ++i) {
                const int j0 = dw.w + BATCH * i;
                if (j0 >= dw.z && !(i == 0 && dw.y == dw.z)) break;
                const int cnt = min(BATCH, dw.z - j0);  // 0 for an empty cluster
                // member indices of rows lane and lane + 32 of the batch
                int t0 = 0, t1 = 0;
                if (lane < cnt) t0 = wc[BATCH * i + lane];
                if (BATCH > 32 && lane + 32 < cnt) t1 = wc[BATCH * i + 32 + lane];
                if (a.rows) {
                    if (lane < cnt) t0 = a.rows[(int64_t)hh * a.L + t0];
                    if (BATCH > 32 && lane + 32 < cnt) t1 = a.rows[(int64_t)hh * a.L + t1];
                }
                const uint32_t slot = it % MS_STAGES;
                if (it >= MS_STAGES && !mbar_wait(bar_empty + 8 * slot, ((it / MS_STAGES) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const uint32_t full = bar_full + 8 * slot;
                if (lane == 0) {
                    const int fl = (j0 == dw.y ? MS_FIRST : 0) | (j0 + BATCH >= dw.z ? MS_LAST : 0) |
                                   (cnt <= 0 ? MS_EMPTY : 0);
                    meta[slot] = make_int4(dw.x, cnt | (fl << 8), dw.z - dw.y, j0);
                }
                const uint32_t dst = sbase + slot * LY::STAGE + (lane % PPR) * 16;
#pragma unroll
                for (int r0 = 0; r0 < BATCH; r0 += RPI) {
                    // the RPI rows of one instruction lie in the same half (r0 is a multiple of RPI)
                    const int r = r0 + lane / PPR;
                    const int tr = __shfl_sync(0xFFFFFFFFu, r0 < 32 ? t0 : t1, r & 31);
                    if (r < cnt) ms_cp16(dst + r * LY::ROWB, src + (int64_t)tr * D);
                }
                const uint32_t ad = sbase + LY::OFF_AUX + (slot * BATCH + lane) * 4;
                if (lane < cnt) {
                    if (MODE == MS_UPDATE_NORM) ms_cp4(ad, a.inv + (int64_t)hh * a.L + t0);
                    if (MODE == MS_STATS) ms_cp4(ad, a.perm + (int64_t)hh * a.L + j0 + lane);
                }
                if (MODE == MS_UPDATE_NORM && BATCH > 32 && lane + 32 < cnt)
                    ms_cp4(ad + 128, a.inv + (int64_t)hh * a.L + t1);
                if (MODE == MS_STATS && cnt > 0 && lane < D / 4) {  // the centre, with every batch
                    const int c = dw.x - hh * a.maxc;
                    ms_cp16(sbase + LY::OFF_CENT + slot * D * 4 + lane * 16,
                            a.C + (int64_t)hh * a.cstride + (int64_t)c * D + lane * 4);
                }
                ms_cp_arrive(full);
                if (lane == 0) mbar_arrive(full);  // publishes meta
                ++it;
            }
        }
        // end marker
        if (ok) {
            const uint32_t slot = it % MS_STAGES;
            if (it >= MS_STAGES && !mbar_wait(bar_empty + 8 * slot, ((it / MS_STAGES) - 1) & 1)) ok = false;
            if (ok) {
                if (lane == 0) meta[slot] = make_int4(0, MS_END << 8, 0, 0);
                ms_cp_arrive(bar_full + 8 * slot);
                if (lane == 0) mbar_arrive(bar_full + 8 * slot);
            }
        }
        if (!ok && lane == 0 && a.err) set_err(a.err, DEV_ERR_TIMEOUT);
        // every copy this warp issued lands before the block exits
        asm volatile("cp.async.wait_all;" ::: "memory");
        return;
    }
    // ---------------- consumers: thread k owns dimension k
    const int k = tid;
    const float *aux_s = reinterpret_cast<const float *>(ms_sm + LY::OFF_AUX);  // inv (update) or token (stats)
    const float *cent_s = reinterpret_cast<const float *>(ms_sm + LY::OFF_CENT);
    constexpr int RS = LY::ROWB / 2;  // row stride in elements
    float s = 0.f, mx = 0.f, mn = 0.f;
    for (uint32_t it = 0;; ++it) {
        const uint32_t slot = it % MS_STAGES;
        if (!mbar_wait(bar_full + 8 * slot, (it / MS_STAGES) & 1)) {
            if (lane == 0 && a.err) set_err(a.err, DEV_ERR_TIMEOUT);
            break;
        }
        const int4 mt = meta[slot];  // cluster, count | flags << 8, members, first position
        const int fl = mt.y >> 8, cnt = mt.y & 0xFF;
        if (fl & MS_END) break;
        const int h = mt.x / a.maxc, c = mt.x - h * a.maxc;
        const uint8_t *rs = ms_sm + slot * LY::STAGE;
        const bf16 *col = reinterpret_cast<const bf16 *>(rs) + k;
        if (MODE != MS_STATS) {
            if (fl & MS_FIRST) s = 0.f;
            const float *inv_s = aux_s + slot * BATCH;
            int r = 0;
            for (; r + 32 <= cnt; r += 32) {
                float v[32];
#pragma unroll
                for (int u = 0; u < 32; ++u) {
                    v[u] = bf2f(col[(r + u) * RS]);
                    if (MODE == MS_UPDATE_NORM) v[u] = __fmul_rn(v[u], inv_s[r + u]);
                }
#pragma unroll
                for (int u = 0; u < 32; ++u) s = __fadd_rn(s, v[u]);
            }
            for (; r < cnt; ++r) {
                float v = bf2f(col[r * RS]);
                if (MODE == MS_UPDATE_NORM) v = __fmul_rn(v, inv_s[r]);
                s = __fadd_rn(s, v);
            }
            if (fl & MS_LAST) {
                const int off = a.coff ? a.coff[h] : 0;
                a.C[(int64_t)h * a.cstride + (int64_t)(off + c) * D + k] = __fdiv_rn(s, (float)mt.z);
            }
        } else {
            const int64_t ci = (int64_t)h * a.maxc + c;
            if (fl & MS_EMPTY) {
                mx = mn = 0.f;
            } else {
                if (fl & MS_FIRST) mx = mn = bf2f(col[0]);
                for (int r = 0; r < cnt; ++r) {
                    const float v = bf2f(col[r * RS]);
                    mx = v > mx ? v : mx;
                    mn = v < mn ? v : mn;
                }
                // the batches take turns among the consumer warps for the
                // exact distances: member row `lane` to the centre
                if (warp == (int)(it % NCW) && lane < cnt) {
                    const int tok = reinterpret_cast<const int *>(aux_s)[slot * BATCH + lane];
                    const float dd = ms_sqdist<D>(rs + lane * LY::ROWB, cent_s + slot * D);
                    a.dmin[(int64_t)h * a.L + tok] = dd;
                    a.dsorted[(int64_t)h * a.L + mt.w + lane] = dd;  // member order, for the SSE
                }
            }
            if (fl & MS_LAST) {
                a.kmax[ci * D + k] = __float2bfloat16(mx);
                a.kmin[ci * D + k] = __float2bfloat16(mn);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty + 8 * slot);
    }
}

template <int D, int MODE>
cudaError_t launch_member_stream(const MsArgs &a, cudaStream_t s) {
    const int total = a.BH * a.maxc;
    if (total <= 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = MsLayout<D, MODE>::BYTES;
    // resident blocks per SM: shared memory (about 220 KB usable), at most 5
    const int per_sm = (int)std::max<size_t>(1, std::min<size_t>(5, (220u << 10) / (smem + 1024)));
    const int G = std::min(total, sms * per_sm);
    cudaError_t e = cudaFuncSetAttribute(k_member_stream<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    k_member_stream<D, MODE><<<G, D + 32, smem, s>>>(a);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_member_stream_d(const MsArgs &a, int d, cudaStream_t s) {
    return d == 128 ? launch_member_stream<128, MODE>(a, s) : launch_member_stream<64, MODE>(a, s);
}

// Per key cluster: count and SSE = the members' exact distances (written in
// member order by the statistics pass) summed in ascending member order; 0
// for the slots c >= n_k.  One warp per cluster: 32 distances per load, the
// next 224 in flight while every lane adds the current ones in order.
__global__ void k_cluster_sse(const int *__restrict__ offs, int offs_stride, const float *__restrict__ dsorted,
                              const int *__restrict__ n_k, int Ccap, int64_t L, int BH, int *__restrict__ counts,
                              float *__restrict__ sse) {
    const int lane = threadIdx.x & 31;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t f = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; f < (int64_t)BH * Ccap; f += nw) {
        const int h = (int)(f / Ccap), c = (int)(f - (int64_t)h * Ccap);
        int beg = 0, end = 0;
        if (c < n_k[h]) {
            beg = offs[(int64_t)h * offs_stride + c];
            end = offs[(int64_t)h * offs_stride + c + 1];
        }
        const float *ds = dsorted + (int64_t)h * L;
        float se = 0.f;
        // eight loads of 32 distances in flight (the largest clusters, thousands
        // of members, would otherwise wait on every load in turn)
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = beg + 32 * u + lane < end ? ds[beg + 32 * u + lane] : 0.f;
        for (int j = beg; j < end; j += 256) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int jb = j + 32 * u;
                if (jb < end) {
                    const int n = min(32, end - jb);
                    const float cur = v[u];
                    v[u] = jb + 256 + lane < end ? ds[jb + 256 + lane] : 0.f;
                    for (int r = 0; r < n; ++r) se = __fadd_rn(se, __shfl_sync(0xFFFFFFFFu, cur, r));
                }
            }
        }
        if (lane == 0) {
            sse[f] = se;
            counts[f] = end - beg;
        }
    }
}

// Bulk copies need 16-byte aligned rows.
inline bool ms_aligned(const bf16 *X) { return (reinterpret_cast<uintptr_t>(X) & 15u) == 0; }

// ------------------------------------------------------------------ update
// Centre = mean of the members, summed in ascending member order in fp32 and
// divided by the count (one thread per dimension).  Normally the members
// stream through k_member_stream below; k_update_direct serves rows that are
// not 16-byte aligned.
// One block per (cluster, unit): each thread loads 32 members ahead from
// global memory.
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
    if (ms_aligned(a.X) && (a.d == 64 || a.d == 128)) {
        MsArgs m{};
        m.X = a.X;
        m.inv = a.inv;
        m.L = a.L;
        m.rows = a.rows;
        m.perm = a.perm;
        m.offs = a.offs;
        m.offs_stride = a.offs_stride;
        m.ncent = a.ncent;
        m.ncent_const = a.ncent_const;
        m.maxc = a.max_cent;
        m.BH = a.BH;
        m.C = a.C;
        m.cstride = a.cstride;
        m.coff = a.coff;
        m.err = a.err;
        return a.inv ? launch_member_stream_d<MS_UPDATE_NORM>(m, a.d, s) : launch_member_stream_d<MS_UPDATE>(m, a.d, s);
    }
    dim3 grid((unsigned)a.max_cent, (unsigned)a.BH);
    if (a.inv) k_update_direct<true><<<grid, a.d, 0, s>>>(a);
    else k_update_direct<false><<<grid, a.d, 0, s>>>(a);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ compensation
// Centroid block of Kp / Vp (ClusterAttention Sec. 1.2): row 8 cgroup + c of unit
// h holds the member means of key cluster c, rounded to bf16; d / 8 threads per
// row and tensor, one block per (cluster, unit).
__global__ void k_comp_rows(const float *__restrict__ kbar, const float *__restrict__ vbar,
                            const int *__restrict__ n_k, int Ccap, int d, int64_t Lpad, int cgroup,
                            bf16 *__restrict__ Kp, bf16 *__restrict__ Vp) {
    const int c = blockIdx.x, h = blockIdx.y;
    if (c >= n_k[h]) return;
    const int per = d / 8, which = threadIdx.x / per, part = threadIdx.x % per;
    const float4 *src = reinterpret_cast<const float4 *>((which ? vbar : kbar) + ((int64_t)h * Ccap + c) * d) + 2 * part;
    const float4 x0 = src[0], x1 = src[1];
    bf16 *dst = (which ? Vp : Kp) + ((int64_t)h * Lpad + (int64_t)cgroup * 8 + c) * d;
    reinterpret_cast<uint4 *>(dst)[part] = make_uint4(pack_bf16x2(x0.x, x0.y), pack_bf16x2(x0.z, x0.w),
                                                      pack_bf16x2(x1.x, x1.y), pack_bf16x2(x1.z, x1.w));
}

cudaError_t launch_comp_rows(const float *kbar, const float *vbar, const int *n_k, int Ccap, int d, int BH,
                             int64_t Lpad, int cgroup, bf16 *Kp, bf16 *Vp, cudaStream_t s) {
    k_comp_rows<<<dim3(Ccap, BH), 2 * (d / 8), 0, s>>>(kbar, vbar, n_k, Ccap, d, Lpad, cgroup, Kp, Vp);
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
    const int64_t pos = stratum_pick(a.seed, (int64_t)a.unit0 + h, a.tag, n, m, j);
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

cudaError_t launch_radix_hist(const float *dist, const int *st_m, int64_t L, int BH, uint32_t *radix, int shift,
                              cudaStream_t s) {
    k_radix_hist<<<dim3(64, BH), 256, 0, s>>>(dist, st_m, L, radix, shift);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
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
// Per key cluster: count, exact per-dimension max/min, and the SSE: the exact
// squared distance of every member to the centre (summed over dimensions in
// order, written to dmin as well), summed over the members in ascending order.
// Normally k_member_stream<MS_STATS> computes them; this one-block-per-cluster
// kernel serves rows that are not 16-byte aligned.
__global__ void k_key_stats(StatsArgs a) {
    const int c = blockIdx.x, h = blockIdx.y, k = threadIdx.x;
    const int nk = a.n_k[h];
    const int64_t ci = (int64_t)h * a.Ccap + c;
    int beg = 0, end = 0;
    if (c < nk) {
        const int *offs = a.offs + (int64_t)h * a.offs_stride;
        beg = offs[c];
        end = offs[c + 1];
    }
    const int *perm = a.perm + (int64_t)h * a.L;
    const bf16 *K = a.K + (int64_t)h * a.L * a.d;
    float mx = 0.f, mn = 0.f;  // an empty cluster keeps 0 (and count 0)
    if (end > beg) mx = mn = bf2f(K[(int64_t)perm[beg] * a.d + k]);
    for (int j = beg + 1; j < end; ++j) {
        const float v = bf2f(K[(int64_t)perm[j] * a.d + k]);
        mx = v > mx ? v : mx;
        mn = v < mn ? v : mn;
    }
    a.kmax[ci * a.d + k] = __float2bfloat16(mx);
    a.kmin[ci * a.d + k] = __float2bfloat16(mn);
    if (k == 0) {
        const float *cc = a.C + (int64_t)h * a.cstride + (int64_t)c * a.d;
        float se = 0.f;
        for (int j = beg; j < end; ++j) {
            const int t = perm[j];
            const bf16 *x = K + (int64_t)t * a.d;
            float acc = 0.f;
            for (int q = 0; q < a.d; ++q) {
                const float tt = __fsub_rn(bf2f(x[q]), cc[q]);
                acc = __fadd_rn(acc, __fmul_rn(tt, tt));
            }
            a.dmin[(int64_t)h * a.L + t] = acc;
            se = __fadd_rn(se, acc);
        }
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
    cudaError_t e;
    if (ms_aligned(a.K) && (a.d == 64 || a.d == 128)) {
        MsArgs m{};
        m.X = a.K;
        m.L = a.L;
        m.perm = a.perm;
        m.offs = a.offs;
        m.offs_stride = a.offs_stride;
        m.ncent = a.n_k;
        m.maxc = a.Ccap;
        m.BH = a.BH;
        m.C = const_cast<float *>(a.C);
        m.cstride = a.cstride;
        m.dmin = a.dmin;
        m.dsorted = a.dsorted;
        m.kmax = a.kmax;
        m.kmin = a.kmin;
        m.err = a.err;
        e = launch_member_stream_d<MS_STATS>(m, a.d, s);
        if (e != cudaSuccess) return e;
        const int64_t n = (int64_t)a.BH * a.Ccap;  // one warp per cluster
        const unsigned blocks = (unsigned)std::min<int64_t>((n + 7) / 8, 148 * 16);
        k_cluster_sse<<<blocks, 256, 0, s>>>(a.offs, a.offs_stride, a.dsorted, a.n_k, a.Ccap, a.L, a.BH, a.counts,
                                             a.sse);
        AC_NOTE_LAUNCH();
        e = cudaGetLastError();
    } else {
        k_key_stats<<<dim3(a.Ccap, a.BH), a.d, 0, s>>>(a);
        AC_NOTE_LAUNCH();
        e = cudaGetLastError();
    }
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
