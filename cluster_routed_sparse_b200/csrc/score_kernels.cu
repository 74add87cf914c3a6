// score_kernels.cu -- critical-cluster selection (AdaCluster, arXiv
// 2604.18348, Sec. 3.2.3 Eq. (1) / Algorithm 2, and Algorithm 3 line 9).
//
// The method's path runs Eq. (1) on the tensor cores, fused with the top-k
// (quest_mma.cu).  The kernels here serve the mean-based ablation
// (score_mode 1) and, on request (AC_EXACT_SCORES=1 at ac_create), Eq. (1) on
// CUDA cores in fp32, each score summed in dimension order, the reference
// arithmetic the tensor-core path reproduces.
// k_quest_scores: one block per (head, 32 key clusters) stages the
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
// clusters -inf.  score_mode 1 (the "w/o Quest" ablation, Sec. 4.4 Table 4)
// stages the cluster's centre mu as both bounds, so the same loop gives
// sum_d q_d mu_d.  Block (h, c-chunk): thread (g, ci) takes key cluster
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
    const bool mean = a.score_mode == 1;
    for (int i = tid; i < a.d * QS_C; i += SEL_THREADS) {
        const int ci = i / a.d, k = i % a.d;  // coalesced over k
        float mx = 0.f, mn = 0.f;
        if (ci < nc) {
            const int64_t o = ((int64_t)h * a.Ccap + c0 + ci) * a.d + k;
            if (mean) {
                mx = mn = a.cent_k[o];  // the mean-based ablation: q_d mu_d
            } else {
                mx = bf2f(a.kmax[o]);
                mn = bf2f(a.kmin[o]);
            }
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
    for (int c = c0; c < c1; ++c)
        if (flag[c]) a.sel[(int64_t)hq * a.Ccap + pos++] = c;
    // The key ranges the attention walks: the kept clusters, or every
    // non-empty cluster of a dense unit (Algorithm 3 line 6), in cluster
    // order, each as (first 8-row group in Kp / Vp, keys); rbox is the
    // exclusive prefix of their 8-row groups.
    const bool dense = a.dense[h] != 0;
    int walk = 0, groups = 0;
    for (int c = c0; c < c1; ++c) {
        const int w = dense ? cnt[c] != 0 : flag[c];
        walk += w;
        groups += w ? (cnt[c] + 7) / 8 : 0;
    }
    __syncthreads();
    int rpos, nr;
    Scan(tmp.scan).ExclusiveSum(walk, rpos, nr);
    __syncthreads();
    int gpos, ng;
    Scan(tmp.scan).ExclusiveSum(groups, gpos, ng);
    __syncthreads();
    const int *pg = a.pgoff + (int64_t)h * a.Ccap;
    int *rbox = a.rbox + (int64_t)hq * (a.Ccap + 1);
    for (int c = c0; c < c1; ++c) {
        const int w = dense ? cnt[c] != 0 : flag[c];
        if (!w) continue;
        a.ranges[(int64_t)hq * a.Ccap + rpos] = make_int2(pg[c], cnt[c]);
        rbox[rpos] = gpos;
        gpos += (cnt[c] + 7) / 8;
        ++rpos;
    }
    // centroid compensation: the unselected non-empty clusters as pseudo-keys
    // (one more range, over the centroid block), with their addends ln|c| / scale
    const bool comp = a.cbias != nullptr && !dense && nonempty > k;
    if (a.cbias) {
        float *cb = a.cbias + (int64_t)hq * a.Ccap;
        for (int c = tid; c < nk; c += SEL_THREADS)
            cb[c] = (flag[c] || cnt[c] == 0) ? -INFINITY : logf((float)cnt[c]) / a.scale;
    }
    if (tid == 0) {
        int n_r = nr, n_g = ng;
        if (comp) {
            a.ranges[(int64_t)hq * a.Ccap + n_r] = make_int2(a.cgroup, nk);
            rbox[n_r] = n_g;
            a.crange[hq] = n_r;
            ++n_r;
            n_g += (nk + 7) / 8;
        } else if (a.crange) {
            a.crange[hq] = -1;
        }
        a.nrange[hq] = n_r;
        a.nboxes[hq] = n_g;
        rbox[n_r] = n_g;
    }
}

// First 8-row group of every key cluster of a unit in Kp / Vp: exclusive
// prefix of ceil(count / 8) in cluster order.  One block per unit.
__global__ void __launch_bounds__(SEL_THREADS) k_group_offsets(const int *counts_k, const int *n_k, int Ccap,
                                                             int *pgoff) {
    typedef cub::BlockScan<int, SEL_THREADS> Scan;
    __shared__ typename Scan::TempStorage tmp;
    const int h = blockIdx.x, tid = threadIdx.x;
    const int nk = n_k[h];
    const int *cnt = counts_k + (int64_t)h * Ccap;
    const int seg = (nk + SEL_THREADS - 1) / SEL_THREADS;
    const int c0 = min(nk, tid * seg), c1 = min(nk, c0 + seg);
    int g = 0;
    for (int c = c0; c < c1; ++c) g += (cnt[c] + 7) / 8;
    int pos;
    Scan(tmp).ExclusiveSum(g, pos);
    for (int c = c0; c < c1; ++c) {
        pgoff[(int64_t)h * Ccap + c] = pos;
        pos += (cnt[c] + 7) / 8;
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

// ------------------------------------------------------------------ tail merging
// Query-tile tail merging (iCATS, "tail merging strategy"), one block per unit.
// Stage 1: a query cluster joins the lowest-index non-empty cluster whose
// selection equals its own (the same key clusters; in a dense unit every
// cluster walks every key, so all join the first); a group's rows are its
// members' rows, member by member in cluster order.  Stage 2 (mode 2, sparse
// units): among the groups with a tail t = rows mod 128 > 0, each finds the
// group whose selection differs from its own in the fewest key clusters
// (ties to the lower index); two groups that are each other's choice and
// whose tails fit one tile pair up: the higher index hands its last t rows to
// the lower, whose key ranges become the union of both selections.
constexpr int TM_TILE = 128;

__device__ __forceinline__ bool tm_same(const int *a, const int *b, int k) {
    for (int i = 0; i < k; ++i)
        if (a[i] != b[i]) return false;
    return true;
}
// |A \ B| + |B \ A| of two ascending lists of k entries
__device__ __forceinline__ int tm_hamming(const int *a, const int *b, int k) {
    int i = 0, j = 0, common = 0;
    while (i < k && j < k) {
        if (a[i] == b[j]) {
            ++common;
            ++i;
            ++j;
        } else if (a[i] < b[j]) {
            ++i;
        } else {
            ++j;
        }
    }
    return 2 * (k - common);
}

__global__ void __launch_bounds__(SEL_THREADS) k_tail_merge_plan(TailMergeArgs a) {
    extern __shared__ int tm_sm[];
    const int Cq = a.Cq, h = blockIdx.x, tid = threadIdx.x;
    int *cnt = tm_sm, *own = cnt + Cq, *S = own + Cq, *tail = S + Cq, *nn = tail + Cq;
    int *partner = nn + Cq, *mv_in = partner + Cq, *mv_out = mv_in + Cq, *offs = mv_out + Cq;  // offs: Cq + 1
    int *pre = offs + Cq + 1;
    const int k = a.ksel[h];
    const bool dense = a.dense[h] != 0;
    const int *sel = a.sel + (int64_t)h * Cq * a.Ccap;
    for (int q = tid; q < Cq; q += SEL_THREADS) {
        cnt[q] = a.counts_q[(int64_t)h * Cq + q];
        S[q] = 0;
        partner[q] = -1;
        mv_in[q] = mv_out[q] = 0;
    }
    __syncthreads();
    // stage 1
    for (int q = tid; q < Cq; q += SEL_THREADS) {
        int o = q;
        if (cnt[q] > 0)
            for (int r = 0; r < q; ++r)
                if (cnt[r] > 0 && (dense || tm_same(sel + (int64_t)r * a.Ccap, sel + (int64_t)q * a.Ccap, k))) {
                    o = r;
                    break;
                }
        own[q] = o;
    }
    __syncthreads();
    for (int q = tid; q < Cq; q += SEL_THREADS)
        if (cnt[q] > 0) atomicAdd(&S[own[q]], cnt[q]);
    __syncthreads();
    // stage 2
    for (int g = tid; g < Cq; g += SEL_THREADS)
        tail[g] = (a.mode >= 2 && !dense && own[g] == g && S[g] > 0) ? S[g] % TM_TILE : 0;
    __syncthreads();
    for (int g = tid; g < Cq; g += SEL_THREADS) {
        int best = -1, bd = 0x7FFFFFFF;
        if (tail[g] > 0)
            for (int o = 0; o < Cq; ++o) {
                if (o == g || tail[o] == 0) continue;
                const int dist = tm_hamming(sel + (int64_t)g * a.Ccap, sel + (int64_t)o * a.Ccap, k);
                if (dist < bd) {
                    bd = dist;
                    best = o;
                }
            }
        nn[g] = best;
    }
    __syncthreads();
    for (int g = tid; g < Cq; g += SEL_THREADS) {
        const int o = nn[g];
        if (tail[g] > 0 && o > g && nn[o] == g && tail[g] + tail[o] <= TM_TILE) {
            partner[g] = o;  // g takes o's tail
            partner[o] = g;
            mv_in[g] = tail[o];
            mv_out[o] = tail[o];
        }
    }
    __syncthreads();
    if (tid == 0) {
        // group offsets (owners only) and every cluster's first position in its group
        int run = 0;
        for (int g = 0; g < Cq; ++g) {
            offs[g] = run;
            run += own[g] == g ? S[g] + mv_in[g] - mv_out[g] : 0;
        }
        offs[Cq] = run;
        for (int g = 0; g < Cq; ++g) nn[g] = 0;  // reused: rows placed so far per group
        for (int q = 0; q < Cq; ++q) {
            pre[q] = nn[own[q]];
            nn[own[q]] += cnt[q];
        }
    }
    __syncthreads();
    int *sc = a.scratch + (int64_t)h * Cq;
    const int64_t plane = (int64_t)a.BH * Cq;
    for (int q = tid; q < Cq; q += SEL_THREADS) {
        const int g = own[q];
        a.counts_qm[(int64_t)h * Cq + q] = own[q] == q ? S[q] + mv_in[q] - mv_out[q] : 0;
        a.offs_qm[(int64_t)h * (Cq + 1) + q] = offs[q];
        sc[q] = g;                                  // owner
        sc[plane + q] = pre[q];                     // first position within the group
        sc[2 * plane + q] = S[q] - mv_out[q];       // rows the group keeps (owners)
        sc[3 * plane + q] = mv_out[q] > 0 ? offs[partner[q]] + S[partner[q]] : 0;  // where handed rows go
    }
    if (tid == 0) a.offs_qm[(int64_t)h * (Cq + 1) + Cq] = offs[Cq];
    // key ranges of the groups that take a tail: the union of both selections, in cluster order
    for (int g = tid; g < Cq; g += SEL_THREADS) {
        if (mv_in[g] == 0) continue;
        const int *A = sel + (int64_t)g * a.Ccap, *B = sel + (int64_t)partner[g] * a.Ccap;
        const int64_t hq = (int64_t)h * Cq + g;
        const int *cntk = a.counts_k + (int64_t)h * a.Ccap;
        const int *pg = a.pgoff + (int64_t)h * a.Ccap;
        int2 *rg = a.ranges + hq * a.Ccap;
        int *rb = a.rbox + hq * (a.Ccap + 1);
        int i = 0, j = 0, nr = 0, box = 0;
        while (i < k || j < k) {
            int c;
            if (j >= k || (i < k && A[i] < B[j])) {
                c = A[i++];
            } else if (i >= k || B[j] < A[i]) {
                c = B[j++];
            } else {
                c = A[i++];
                ++j;
            }
            rg[nr] = make_int2(pg[c], cntk[c]);
            rb[nr] = box;
            box += (cntk[c] + 7) / 8;
            ++nr;
        }
        rb[nr] = box;
        a.nrange[hq] = nr;
        a.nboxes[hq] = box;
    }
}

// Rows of Qp in group order: the row at cluster-order position p (cluster q,
// i-th member) goes to its group's position pre[q] + i, or, past the rows the
// group keeps, to the group that takes its tail.
__global__ void k_tail_merge_perm(TailMergeArgs a) {
    const int h = blockIdx.y;
    const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= a.L) return;
    const int64_t plane = (int64_t)a.BH * a.Cq;
    const int tok = a.perm_q[(int64_t)h * a.L + p];
    const int q = a.labels_q[(int64_t)h * a.L + tok];
    const int *sc = a.scratch + (int64_t)h * a.Cq;
    const int g = sc[q];
    const int gp = sc[plane + q] + (int)(p - a.offs_q[(int64_t)h * (a.Cq + 1) + q]);
    const int keep = sc[2 * plane + g];
    const int dest = gp < keep ? a.offs_qm[(int64_t)h * (a.Cq + 1) + g] + gp : sc[3 * plane + g] + (gp - keep);
    a.perm_qm[(int64_t)h * a.L + dest] = tok;
}

cudaError_t launch_tail_merge(const TailMergeArgs &a, cudaStream_t s) {
    const size_t smem = (size_t)(10 * a.Cq + 1) * sizeof(int);
    cudaError_t e;
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(k_tail_merge_plan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_tail_merge_plan<<<a.BH, SEL_THREADS, smem, s>>>(a);
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_tail_merge_perm<<<dim3((unsigned)((a.L + 255) / 256), a.BH), 256, 0, s>>>(a);
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_tile_prefix<<<1, 1024, 0, s>>>(a.counts_qm, a.BH * a.Cq, a.tile_prefix);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

cudaError_t launch_score_select(const SelectArgs &a, cudaStream_t s) {
    cudaError_t e;
    if (!a.exact_cuda_cores && quest_mma_supported(a)) {
        // Eq. (1) on the tensor cores fused with the top-k and the key ranges
        // (quest_mma.cu); it needs each cluster's first 8-row group first
        k_group_offsets<<<a.BH, SEL_THREADS, 0, s>>>(a.counts_k, a.n_k, a.Ccap, a.pgoff);
        AC_NOTE_LAUNCH();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = launch_quest_select_mma(a, s)) != cudaSuccess) return e;
        k_tile_prefix<<<1, 1024, 0, s>>>(a.counts_q, a.BH * a.Cq, a.tile_prefix);
        AC_NOTE_LAUNCH();
        return cudaGetLastError();
    }
    const size_t qsm = (size_t)(2 * a.d * QS_C + a.Cq * a.d) * 4;
    if (qsm > 200 * 1024) return cudaErrorInvalidValue;  // ac_create keeps Cq within this
    e = cudaFuncSetAttribute(k_quest_scores, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(qsm < 48 * 1024 ? 48 * 1024 : qsm));
    if (e != cudaSuccess) return e;
    k_quest_scores<<<dim3((a.Ccap + QS_C - 1) / QS_C, a.BH), SEL_THREADS, qsm, s>>>(a);
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    size_t smem = (size_t)a.Ccap * 4 * 2;
    e = cudaFuncSetAttribute(k_score_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(smem < 48 * 1024 ? 48 * 1024 : smem));
    if (e != cudaSuccess) return e;
    k_group_offsets<<<a.BH, SEL_THREADS, 0, s>>>(a.counts_k, a.n_k, a.Ccap, a.pgoff);
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_score_select<<<a.BH * a.Cq, SEL_THREADS, smem, s>>>(a);
    AC_NOTE_LAUNCH();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_tile_prefix<<<1, 1024, 0, s>>>(a.counts_q, a.BH * a.Cq, a.tile_prefix);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

}  // namespace ac
