// score_kernels.cu -- critical-cluster selection (AdaCluster, arXiv
// 2604.18348, Sec. 3.2.3 Eq. (1) / Algorithm 2, and Algorithm 3 line 9).
//
// At cluster granularity the score matrix of one head is Cq x n_k (65 x ~1000)
// over d = 128: about 17 MFLOP per head, far too small to fill the tensor
// cores of one SM, so one block per (head, query cluster) computes its row of
// Eq. (1) on CUDA cores in fp32, summed in dimension order, and selects the
// top-k in the same block.  The selection is exact: every score is compared in
// the precision and order it was formed in.
#include <cub/block/block_reduce.cuh>
#include <cub/block/block_scan.cuh>

#include "ac_device.cuh"
#include "ac_internal.h"

namespace ac {

constexpr int SEL_THREADS = 256;

__global__ void __launch_bounds__(SEL_THREADS) k_score_select(SelectArgs a) {
    extern __shared__ __align__(16) float sm[];
    float *S = sm;               // [Ccap]
    float *q = sm + a.Ccap;      // [d]
    int *flag = reinterpret_cast<int *>(q + a.d);  // [Ccap]
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
    for (int k = tid; k < a.d; k += SEL_THREADS) q[k] = a.cent_q[(int64_t)hq * a.d + k];
    __syncthreads();

    // Eq. (1): S[c] = sum_d max(q_d * Kmax_d, q_d * Kmin_d); empty clusters -inf.
    int ne = 0;
    for (int c = tid; c < nk; c += SEL_THREADS) {
        float s;
        if (cnt[c] == 0) {
            s = -INFINITY;
        } else {
            ++ne;
            const bf16 *mx = a.kmax + ((int64_t)h * a.Ccap + c) * a.d;
            const bf16 *mn = a.kmin + ((int64_t)h * a.Ccap + c) * a.d;
            s = 0.f;
            for (int k = 0; k < a.d; ++k) {
                float u = __fmul_rn(q[k], bf2f(mx[k]));
                float v = __fmul_rn(q[k], bf2f(mn[k]));
                s = __fadd_rn(s, u > v ? u : v);
            }
        }
        S[c] = s;
        a.score[(int64_t)hq * a.Ccap + c] = s;
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

    // Rank of each cluster in (score desc, id asc) order; the k first are kept.
    const int seg = (nk + SEL_THREADS - 1) / SEL_THREADS;
    const int c0 = min(nk, tid * seg), c1 = min(nk, c0 + seg);
    int mine = 0;
    for (int c = c0; c < c1; ++c) {
        const float sc = S[c];
        int take = 0;
        if (sc != -INFINITY) {
            int rank = 0;
            for (int o = 0; o < nk; ++o) {
                const float so = S[o];
                rank += (so > sc) || (so == sc && o < c);
            }
            take = rank < k;
        }
        flag[c] = take;
        mine += take;
    }
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
    size_t smem = (size_t)a.Ccap * 4 * 2 + (size_t)a.d * 4;
    cudaError_t e = cudaFuncSetAttribute(k_score_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
