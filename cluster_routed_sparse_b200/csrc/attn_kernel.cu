// attn_kernel.cu -- exact softmax attention over the selected key clusters
// (AdaCluster, arXiv 2604.18348, Algorithm 3 lines 5-11) on tcgen05 / TMEM.
//
// Inputs are the cluster-order copies Qp, Kp, Vp ([BH*L, d] bf16): the queries
// of one query cluster are contiguous, and so are the keys of one key cluster.
// One CTA handles one 128-query tile of one query cluster.  Its key set is the
// list of row ranges of the selected key clusters (one range of all L keys for
// a dense unit), walked in 8-row boxes; 16 boxes form a 128-column key tile.
// Columns of a box past the end of its cluster are masked, so a cluster wastes
// at most 7 columns.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread t owns query row t = TMEM lane t
//   warp 4     TMA producer (Q tile once; K and V boxes per key tile)
//   warp 5     TMEM allocator and the single-thread tcgen05.mma issuer
// Pipeline per key tile j (S and O double-buffered in TMEM, K/V in 2 stages):
//   S_j = Q K_j^T  -> softmax_j (P_j to smem)  -> O_j = P_j V_j
// with S_{j+1} issued before PV_j, so the tensor core runs while the softmax
// warps work.  The softmax warps keep the output row in registers:
//   acc = acc * 2^(m_{j-1} - m_j) + O_j.
// Every mbarrier wait is bounded; on timeout the CTA records an error, drains
// what it issued and frees its TMEM.
#include "ac_device.cuh"
#include "ac_internal.h"

namespace ac {
namespace {

constexpr int BM = 128;       // query rows per tile
constexpr int BN = 128;       // key columns per tile
constexpr int NS = 2;         // K/V pipeline stages
constexpr int BOXES = BN / 8; // 8-row boxes per key tile
constexpr int NTHREADS = 192;

template <int D>
struct Layout {
    static constexpr int HALVES = D / 64;  // 128-byte (64 x bf16) column halves
    static constexpr uint32_t Q_BYTES = HALVES * BM * 128;
    static constexpr uint32_t KV_BYTES = HALVES * BN * 128;
    static constexpr uint32_t P_BYTES = 2 * BM * 128;  // 128 keys = 2 halves
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + NS * KV_BYTES;
    static constexpr uint32_t OFF_P = OFF_V + NS * KV_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_P + 2 * P_BYTES;
    static constexpr uint32_t BYTES = OFF_BAR + 256;
    static constexpr uint32_t SMEM = BYTES + 1024;  // 1024-byte alignment slack
};

enum {
    B_KVF = 0,   // [2] K/V stage filled (TMA tx)
    B_KVE = 2,   // [2] K/V stage free (MMA commit)
    B_QF = 4,    // Q tile filled
    B_SF = 5,    // [2] S buffer written (MMA commit)
    B_SE = 7,    // [2] S buffer read (128 softmax threads)
    B_PF = 9,    // [2] P buffer written (128 softmax threads)
    B_OF = 11,   // [2] O buffer written (MMA commit)
    B_OE = 13,   // [2] O buffer read (128 softmax threads)
    B_DONE = 15, // all MMAs complete
    NBAR = 16
};

struct KeyWalker {
    const int2 *rg;
    int nr, r, o;
    __device__ __forceinline__ void init(const int2 *g, int n) {
        rg = g;
        nr = n;
        r = 0;
        o = 0;
    }
    // Next 8-row box: first row (within the unit) and number of valid rows.
    __device__ __forceinline__ void next(int &start, int &cnt) {
        if (r < nr) {
            const int2 g = rg[r];
            start = g.x + o;
            const int rem = g.y - o;
            cnt = rem < 8 ? rem : 8;
            o += cnt;
            if (o >= g.y) {
                ++r;
                o = 0;
            }
        } else {
            start = 0;
            cnt = 0;
        }
    }
};

struct AttnParams {
    bf16 *O;
    const int *perm_q, *offs_q, *counts_q, *tile_prefix, *nboxes, *ksel;
    const int2 *ranges;
    const uint8_t *dense;
    int L, Cq, Ccap, BH;
    float scale_log2;
    uint32_t *err;
    unsigned long long *counters;
};

// acc = acc * a + O_jj (row of this thread), then release the O buffer.
template <int D>
__device__ __forceinline__ bool accumulate_o(float (&acc)[D], uint32_t tmem_row, uint32_t bar_full,
                                             uint32_t bar_empty, int jj, float a) {
    if (!mbar_wait(bar_full, (jj >> 1) & 1)) return false;
    tc_fence_after();
    const uint32_t tO = tmem_row + 256 + (jj & 1) * 128;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[c * 32 + i] = acc[c * 32 + i] * a + __uint_as_float(r[i]);
    }
    tc_fence_before();
    mbar_arrive(bar_empty);
    return true;
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_sparse_attn(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
    using LY = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- work item: (unit h, query cluster qc, 128-row tile)
    const int nhq = p.BH * p.Cq;
    const int item = blockIdx.x;
    if (item >= p.tile_prefix[nhq]) return;
    int lo = 0, hi = nhq;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.tile_prefix[mid] <= item) lo = mid;
        else hi = mid;
    }
    const int hq = lo, h = hq / p.Cq, qc = hq % p.Cq;
    const int tile = item - p.tile_prefix[hq];
    const int row0 = p.offs_q[(int64_t)h * (p.Cq + 1) + qc] + tile * BM;
    const int nvalid = min(BM, p.counts_q[hq] - tile * BM);
    const int64_t unit_row = (int64_t)h * p.L;
    const int n_tiles = (p.nboxes[hq] + BOXES - 1) / BOXES;
    const int2 *rg = p.ranges + (int64_t)hq * p.Ccap;
    const int nr = p.dense[h] ? 1 : p.ksel[h];

    const uint32_t bar0 = sbase + LY::OFF_BAR;
#define BAR(i) (bar0 + 8u * (uint32_t)(i))
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + LY::OFF_BAR + 8 * NBAR);

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(B_KVF + i), 1);
            mbar_init(BAR(B_KVE + i), 1);
            mbar_init(BAR(B_SF + i), 1);
            mbar_init(BAR(B_SE + i), BM);
            mbar_init(BAR(B_PF + i), BM);
            mbar_init(BAR(B_OF + i), 1);
            mbar_init(BAR(B_OE + i), BM);
        }
        mbar_init(BAR(B_QF), 1);
        mbar_init(BAR(B_DONE), 1);
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 4) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            mbar_arrive_expect_tx(BAR(B_QF), LY::Q_BYTES);
            for (int hf = 0; hf < LY::HALVES; ++hf)
                tma_load_2d(sbase + LY::OFF_Q + hf * BM * 128, &tm_q, hf * 64, (int)(unit_row + row0),
                            BAR(B_QF));
            KeyWalker w;
            w.init(rg, nr);
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % NS;
                if (j >= NS && !mbar_wait(BAR(B_KVE + s), ((j / NS) - 1) & 1)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(BAR(B_KVF + s), 2 * LY::KV_BYTES);
                const uint32_t kd = sbase + LY::OFF_K + s * LY::KV_BYTES;
                const uint32_t vd = sbase + LY::OFF_V + s * LY::KV_BYTES;
                for (int b = 0; b < BOXES; ++b) {
                    int st, c;
                    w.next(st, c);
                    const int row = (int)(unit_row + st);
                    for (int hf = 0; hf < LY::HALVES; ++hf) {
                        tma_load_2d(kd + hf * BN * 128 + b * 1024, &tm_k, hf * 64, row, BAR(B_KVF + s));
                        tma_load_2d(vd + hf * BN * 128 + b * 1024, &tm_v, hf * 64, row, BAR(B_KVF + s));
                    }
                }
                ++issued;
            }
            // Loads still in flight must land before the CTA exits.
            for (int j = issued - NS < 0 ? 0 : issued - NS; j < issued; ++j)
                if (!mbar_wait(BAR(B_KVF + (j % NS)), (j / NS) & 1)) ok = false;
            if (!mbar_wait(BAR(B_QF), 0)) ok = false;
            if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 5) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IQK = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t IPV = idesc_bf16_f32(BM, D, true);
            const uint32_t qa = sbase + LY::OFF_Q;
            if (!mbar_wait(BAR(B_QF), 0)) ok = false;
            tc_fence_after();
            auto issue_s = [&](int j) -> bool {
                const int s = j % NS, b = j & 1;
                if (!mbar_wait(BAR(B_KVF + s), (j / NS) & 1)) return false;
                if (j >= 2 && !mbar_wait(BAR(B_SE + b), ((j >> 1) - 1) & 1)) return false;
                tc_fence_after();
                const uint32_t ka = sbase + LY::OFF_K + s * LY::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    tc_mma_bf16(tmem + b * BN, sdesc_sw128(qa + off, 16, 1024),
                                sdesc_sw128(ka + off, 16, 1024), IQK, kk > 0 ? 1u : 0u);
                }
                tc_commit(BAR(B_SF + b));
                return true;
            };
            if (ok && n_tiles > 0) ok = issue_s(0);
            for (int j = 0; j < n_tiles && ok; ++j) {
                if (j + 1 < n_tiles && !issue_s(j + 1)) {
                    ok = false;
                    break;
                }
                const int s = j % NS, b = j & 1;
                if (!mbar_wait(BAR(B_PF + b), (j >> 1) & 1)) {
                    ok = false;
                    break;
                }
                if (j >= 2 && !mbar_wait(BAR(B_OE + b), ((j >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t pa = sbase + LY::OFF_P + b * LY::P_BYTES;
                const uint32_t va = sbase + LY::OFF_V + s * LY::KV_BYTES;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint32_t aoff = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    const uint32_t boff = kk * 16 * 128;
                    tc_mma_bf16(tmem + 256 + b * 128, sdesc_sw128(pa + aoff, 16, 1024),
                                sdesc_sw128(va + boff, BN * 128, 1024), IPV, kk > 0 ? 1u : 0u);
                }
                tc_commit(BAR(B_OF + b));
                tc_commit(BAR(B_KVE + s));
            }
            tc_commit(BAR(B_DONE));
            if (!mbar_wait(BAR(B_DONE), 0)) ok = false;
            if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ softmax + epilogue
        const int row = tid;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float sl2 = p.scale_log2;
        float m_run = -INFINITY, l_run = 0.f, alpha_prev = 0.f;
        float acc[D];
#pragma unroll
        for (int k = 0; k < D; ++k) acc[k] = 0.f;
        long long kept_cols = 0;

        KeyWalker w;
        w.init(rg, nr);
        for (int j = 0; j < n_tiles; ++j) {
            uint32_t vm[4] = {0u, 0u, 0u, 0u};
#pragma unroll 1
            for (int bx = 0; bx < BOXES; ++bx) {
                int st, c;
                w.next(st, c);
                const uint32_t bits = c >= 8 ? 0xFFu : ((1u << c) - 1u);
                vm[bx >> 2] |= bits << ((bx & 3) * 8);
            }
            kept_cols += __popc(vm[0]) + __popc(vm[1]) + __popc(vm[2]) + __popc(vm[3]);
            const int b = j & 1;
            if (!mbar_wait(BAR(B_SF + b), (j >> 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tS = tmem + lane_off + b * BN;
            float tmax = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(tS + c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if ((vm[c] >> i) & 1u) tmax = fmaxf(tmax, __uint_as_float(r[i]));
            }
            const float m_new = fmaxf(m_run, tmax * sl2);
            const float alpha = ex2_approx(m_run - m_new);
            float rs = 0.f;
            uint8_t *pb = sm + LY::OFF_P + b * LY::P_BYTES;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(tS + c * 32, r);
                tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    const float p0 = ((vm[c] >> i) & 1u) ? ex2_approx(__uint_as_float(r[i]) * sl2 - m_new) : 0.f;
                    const float p1 =
                        ((vm[c] >> (i + 1)) & 1u) ? ex2_approx(__uint_as_float(r[i + 1]) * sl2 - m_new) : 0.f;
                    rs += p0 + p1;
                    pk[i >> 1] = pack_bf16x2(p0, p1);
                }
                // keys [32c, 32c+32): half c>>1, 16-byte chunks (c&1)*4 .. +3, 128B swizzle
                uint8_t *rowp = pb + (c >> 1) * (BM * 128) + row * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int chunk = (((c & 1) * 4) + q4) ^ (row & 7);
                    *reinterpret_cast<uint4 *>(rowp + chunk * 16) =
                        make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(BAR(B_SE + b));
            fence_proxy_async_smem();
            mbar_arrive(BAR(B_PF + b));
            l_run = l_run * alpha + rs;
            m_run = m_new;
            if (j >= 1 && !accumulate_o<D>(acc, tmem + lane_off, BAR(B_OF + ((j - 1) & 1)),
                                           BAR(B_OE + ((j - 1) & 1)), j - 1, alpha_prev)) {
                ok = false;
                break;
            }
            alpha_prev = alpha;
        }
        if (ok && n_tiles > 0 &&
            !accumulate_o<D>(acc, tmem + lane_off, BAR(B_OF + ((n_tiles - 1) & 1)), BAR(B_OE + ((n_tiles - 1) & 1)),
                             n_tiles - 1, alpha_prev))
            ok = false;
        if (!ok) {
            set_err(p.err, DEV_ERR_TIMEOUT);
        } else if (row < nvalid) {
            const float il = n_tiles > 0 ? 1.f / l_run : 0.f;
            const int tok = p.perm_q[unit_row + row0 + row];
            uint4 *dst = reinterpret_cast<uint4 *>(p.O + (unit_row + tok) * D);
#pragma unroll
            for (int k8 = 0; k8 < D / 8; ++k8)
                dst[k8] = make_uint4(pack_bf16x2(acc[8 * k8] * il, acc[8 * k8 + 1] * il),
                                     pack_bf16x2(acc[8 * k8 + 2] * il, acc[8 * k8 + 3] * il),
                                     pack_bf16x2(acc[8 * k8 + 4] * il, acc[8 * k8 + 5] * il),
                                     pack_bf16x2(acc[8 * k8 + 6] * il, acc[8 * k8 + 7] * il));
        }
        if (tid == 0 && p.counters) {
            atomicAdd(&p.counters[0], (unsigned long long)((long long)nvalid * kept_cols));
            atomicAdd(&p.counters[1], (unsigned long long)((long long)BM * BN * n_tiles));
            atomicAdd(&p.counters[2], 1ull);
        }
    }
#undef BAR
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

int attn_max_tiles(int L, int Cq, int BH) { return BH * ((L + BM - 1) / BM + Cq); }

cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t s) {
    AttnParams p;
    p.O = a.O;
    p.perm_q = a.perm_q;
    p.offs_q = a.offs_q;
    p.counts_q = a.counts_q;
    p.tile_prefix = a.tile_prefix;
    p.nboxes = a.nboxes;
    p.ksel = a.ksel;
    p.ranges = a.ranges;
    p.dense = a.dense;
    p.L = a.L;
    p.Cq = a.Cq;
    p.Ccap = a.Ccap;
    p.BH = a.BH;
    p.scale_log2 = a.scale_log2;
    p.err = a.err;
    p.counters = a.counters;
    const int grid = attn_max_tiles(a.L, a.Cq, a.BH);
    cudaError_t e;
    if (a.d == 128) {
        e = cudaFuncSetAttribute(k_sparse_attn<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Layout<128>::SMEM);
        if (e != cudaSuccess) return e;
        k_sparse_attn<128><<<grid, NTHREADS, Layout<128>::SMEM, s>>>(*a.tm_q, *a.tm_k, *a.tm_v, p);
        AC_NOTE_LAUNCH();
    } else {
        e = cudaFuncSetAttribute(k_sparse_attn<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Layout<64>::SMEM);
        if (e != cudaSuccess) return e;
        k_sparse_attn<64><<<grid, NTHREADS, Layout<64>::SMEM, s>>>(*a.tm_q, *a.tm_k, *a.tm_v, p);
        AC_NOTE_LAUNCH();
    }
    return cudaGetLastError();
}

}  // namespace ac
