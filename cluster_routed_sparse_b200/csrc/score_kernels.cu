// score_kernels.cu -- critical-cluster selection (AdaCluster, arXiv
// 2604.18348, Sec. 3.2.3 Eq. (1) / Algorithm 2, and Algorithm 3 line 9).
//
// At cluster granularity the score matrix of one head is Cq x n_k (65 x ~1000)
// over d = 128: about 17 MFLOP per head, far too small to fill the tensor
// cores, so it runs on CUDA cores in fp32, each score summed in dimension
// order.  k_quest_scores: one block per (head, 32 key clusters) stages the
// clusters' bounds and all query centroids in shared memory, each thread
// accumulating the scores of one key cluster against 9 query centroids per
// pass.
// k_select: one block per (head, query cluster) selects the top-k of its row.
// The selection is exact: every score is compared in the precision and order
// it was formed in.
#include <cub/block/block_reduce.cuh>
#include <cub/block/block_scan.cuh>

#include "ac_device.cuh"
#include "ac_internal.h"

namespace ac {

constexpr int SEL_THREADS = 256;

constexpr int QS_C = 32;                        // key clusters per block
constexpr int QS_G = SEL_THREADS / QS_C;        // query-centroid groups
constexpr int QS_PER = 9;                       // query centroids per thread and pass

// Eq. (1) for every (query cluster, key cluster) of a head:
//   S[qc, c] = sum_d max(q_d Kmax_d, q_d Kmin_d), summed d = 0, 1, ...; empty
// clusters -inf.  Block (h, c-chunk): thread (g, ci) takes key cluster
// c0 + ci against query centroids g, g + QS_G, ...  Bounds stored [d][32]
// (conflict-free), centroids [Cq][d] (broadcast within a warp).
__global__ void __launch_bounds__(SEL_THREADS) k_quest_scores(SelectArgs a) {
    extern __shared__ __align__(16) float qs_sm[];
    float *kx = qs_sm;                    // [d][QS_C]
    float *kn = kx + a.d * QS_C;          // [d][QS_C]
    float *qv = kn + a.d * QS_C;          // [Cq][d]
    const int h = blockIdx.y, c0 = blockIdx.x * QS_C, tid = threadIdx.x;
    const int nk = a.n_k[h];
    if (c0 >= nk) return;
    const int nc = min(QS_C, nk - c0);
    for (int i = tid; i < a.d * QS_C; i += SEL_THREADS) {
        const int ci = i / a.d, k = i % a.d;  // coalesced over k
        float mx = 0.f, mn = 0.f;
        if (ci < nc) {
            const int64_t o = ((int64_t)h * a.Ccap + c0 + ci) * a.d + k;
            mx = bf2f(a.kmax[o]);
            mn = bf2f(a.kmin[o]);
        }
        kx[k * QS_C + ci] = mx;
        kn[k * QS_C + ci] = mn;
    }
    for (int i = tid; i < a.Cq * a.d; i += SEL_THREADS) qv[i] = a.cent_q[(int64_t)h * a.Cq * a.d + i];
    __syncthreads();
    const int ci = tid % QS_C, g = tid / QS_C;
    const bool empty = ci < nc && a.counts_k[(int64_t)h * a.Ccap + c0 + ci] == 0;
    for (int qb = 0; qb < a.Cq; qb += QS_G * QS_PER) {
        float acc[QS_PER];
#pragma unroll
        for (int j = 0; j < QS_PER; ++j) acc[j] = 0.f;
        for (int k = 0; k < a.d; ++k) {
            const float mx = kx[k * QS_C + ci], mn = kn[k * QS_C + ci];
#pragma unroll
            for (int j = 0; j < QS_PER; ++j) {
                const int qc = qb + g + QS_G * j;
                if (qc < a.Cq) {
                    const float qd = qv[qc * a.d + k];
                    const float u = __fmul_rn(qd, mx);
                    const float v = __fmul_rn(qd, mn);
                    acc[j] = __fadd_rn(acc[j], u > v ? u : v);
                }
            }
        }
        if (ci < nc) {
#pragma unroll
            for (int j = 0; j < QS_PER; ++j) {
                const int qc = qb + g + QS_G * j;
                if (qc < a.Cq) a.score[((int64_t)h * a.Cq + qc) * a.Ccap + c0 + ci] = empty ? -INFINITY : acc[j];
            }
        }
    }
}

__global__ void __launch_bounds__(SEL_THREADS) k_score_select(SelectArgs a) {
    extern __shared__ __align__(16) float sm[];
    float *S = sm;               // [Ccap]
    int *flag = reinterpret_cast<int *>(sm + a.Ccap);  // [Ccap]
    typedef cub::BlockScan<int, SEL_THREADS> Scan;
    typedef cub::BlockReduce<int, SEL_THREADS> Red;
    __shared__ union {
        typename Scan::TempStorage scan;
        typename Red::TempStorage red;
    } tmp;
    __shared__ int k_s;

    const int hq = blockIdx.x, h = hq / a.Cq, qc = hq % a.Cq, tid = threadIdx.x;
    const int nk = a.n_k[h];
    const int *cnt = a.counts_k + (int64_t)h * a.Ccap;

    // this row of Eq. (1) (k_quest_scores); empty clusters are -inf
    int ne = 0;
    for (int c = tid; c < nk; c += SEL_THREADS) {
        const float sc = a.score[(int64_t)hq * a.Ccap + c];
        S[c] = sc;
        ne += cnt[c] != 0;
    }
    const int nonempty = Red(tmp.red).Sum(ne);
    if (tid == 0) {
        int64_t k = a.topk > 0 ? a.topk : ((int64_t)(-a.topk) * nk + 999) / 1000;
        if (k > nonempty) k = nonempty;
        if (k < 1) k = 1;
        k_s = (int)k;
        if (qc == 0) a.ksel[h] = (int)k;
    }
    __syncthreads();
    const int k = k_s;

    // The k first clusters in (score desc, id asc) order are kept.  Radix
    // select (8-bit digits, most significant first) finds the k-th largest
    // score key K*; every cluster above K* is kept, and of those equal to K*
    // the ones with the lowest ids.  Keys order the fp32 scores (both zeros
    // map to one key, as they compare equal); empty clusters take no part.
    unsigned int *key = reinterpret_cast<unsigned int *>(flag);  // reused: key, then the flag
    for (int c = tid; c < nk; c += SEL_THREADS) {
        const float sc = S[c];
        const uint32_t u = __float_as_uint(sc == 0.f ? 0.f : sc);
        key[c] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    __shared__ unsigned int hist[256];
    __shared__ unsigned int sel_prefix, sel_above;
    if (tid == 0) {
        sel_prefix = 0u;
        sel_above = 0u;
    }
    for (int shift = 24; shift >= 0; shift -= 8) {
        hist[tid] = 0u;  // SEL_THREADS == 256
        __syncthreads();
        const unsigned int pre = sel_prefix;
        for (int c = tid; c < nk; c += SEL_THREADS) {
            if (S[c] == -INFINITY) continue;
            const unsigned int kc = key[c];
            if (shift == 24 || (kc >> (shift + 8)) == pre) atomicAdd(&hist[(kc >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid == 0) {
            const unsigned int need = (unsigned int)k - sel_above;
            unsigned int cum = 0u;
            int dg = 255;
            for (; dg > 0; --dg) {
                if (cum + hist[dg] >= need) break;
                cum += hist[dg];
            }
            sel_above += cum;
            sel_prefix = (pre << 8) | (unsigned int)dg;
        }
        __syncthreads();
    }
    const unsigned int kstar = sel_prefix;
    const int need_eq = k - (int)sel_above;
    const int seg = (nk + SEL_THREADS - 1) / SEL_THREADS;
    const int c0 = min(nk, tid * seg), c1 = min(nk, c0 + seg);
    int eq = 0;
    for (int c = c0; c < c1; ++c) eq += (S[c] != -INFINITY && key[c] == kstar);
    int eq_before;
    Scan(tmp.scan).ExclusiveSum(eq, eq_before);
    __syncthreads();
    int mine = 0;
    for (int c = c0; c < c1; ++c) {
        int take = 0;
        if (S[c] != -INFINITY) {
            const unsigned int kc = key[c];
            if (kc > kstar) take = 1;
            else if (kc == kstar) take = eq_before++ < need_eq;
        }
        mine += take;
        key[c] = (unsigned int)take;  // the flag from here on
    }
    __syncthreads();
    int pos;
    Scan(tmp.scan).ExclusiveSum(mine, pos);
    __syncthreads();
    // 8-row boxes of the kept clusters: exclusive prefix in selection order
    int boxes = 0;
    for (int c = c0; c < c1; ++c)
        if (flag[c]) boxes += (cnt[c] + 7) / 8;
    int bpos, nb;
    Scan(tmp.scan).ExclusiveSum(boxes, bpos, nb);
    __syncthreads();
    const int *offs = a.offs_k + (int64_t)h * (a.Ccap + 1);
    int *rbox = a.rbox + (int64_t)hq * (a.Ccap + 1);
    for (int c = c0; c < c1; ++c) {
        if (!flag[c]) continue;
        a.sel[(int64_t)hq * a.Ccap + pos] = c;
        a.ranges[(int64_t)hq * a.Ccap + pos] = make_int2(offs[c], cnt[c]);
        rbox[pos] = bpos;
        bpos += (cnt[c] + 7) / 8;
        ++pos;
    }
    __syncthreads();
    if (tid == 0) {
        if (a.dense[h]) {  // Algorithm 3 line 6: every key of the unit
            a.ranges[(int64_t)hq * a.Ccap] = make_int2(0, a.L);
            a.nboxes[hq] = (a.L + 7) / 8;
            rbox[0] = 0;
            rbox[1] = (a.L + 7) / 8;
        } else {
            a.nboxes[hq] = nb;
            rbox[k] = nb;
        }
    }
}

// Exclusive prefix of the number of attention work items of every (unit, query
// cluster): one item per pair of 128-query tiles.
__global__ void __launch_bounds__(1024) k_tile_prefix(const int *counts_q, int n, int *prefix) {
    typedef cub::BlockScan<int, 1024> Scan;
    __shared__ typename Scan::TempStorage tmp;
    __shared__ int base_s;
    if (threadIdx.x == 0) base_s = 0;
    __syncthreads();
    for (int i0 = 0; i0 < n; i0 += 1024) {
        const int i = i0 + threadIdx.x;
        const int t = i < n ? (counts_q[i] + 255) / 256 : 0;
        int p, tot;
        Scan(tmp).ExclusiveSum(t, p, tot);
        const int base = base_s;
        if (i < n) prefix[i] = base + p;
        __syncthreads();
        if (threadIdx.x == 0) base_s = base + tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) prefix[n] = base_s;
}

cudaError_t launch_score_select(const SelectArgs &a, cudaStream_t s) {
    const size_t qsm = (size_t)(2 * a.d * QS_C + a.Cq * a.d) * 4;
    if (qsm > 200 * 1024) return cudaErrorInvalidValue;  // ac_create keeps Cq within this
    cudaError_t e = cudaFuncSetAttribute(k_quest_scores, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(qsm < 48 * 1024 ? 48 * 1024 : qsm));
    if (e != cudaSuccess) return e;
    k_quest_scores<<<dim3((a.Ccap + QS_C - 1) / QS_C, a.BH), SEL_THREADS, qsm, s>>>(a);
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    size_t smem = (size_t)a.Ccap * 4 * 2;
    e = cudaFuncSetAttribute(k_score_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(smem < 48 * 1024 ? 48 * 1024 : smem));
    if (e != cudaSuccess) return e;
    k_score_select<<<a.BH * a.Cq, SEL_THREADS, smem, s>>>(a);
    AC_NOTE_LAUNCH();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_tile_prefix<<<1, 1024, 0, s>>>(a.counts_q, a.BH * a.Cq, a.tile_prefix);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

}  // namespace ac
