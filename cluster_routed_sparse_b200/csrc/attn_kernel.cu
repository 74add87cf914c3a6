// attn_kernel.cu -- exact softmax attention over the selected key clusters
// (AdaCluster, arXiv 2604.18348, Algorithm 3 lines 5-11) on tcgen05 / TMEM.
//
// Inputs are the cluster-order copies Qp, Kp, Vp ([BH*L, d] bf16): the queries
// of one query cluster are contiguous, and so are the keys of one key cluster.
// One CTA handles two consecutive 128-query tiles of one query cluster, which
// share every K/V tile.  The key set is the list of row ranges of the selected
// key clusters (one range of all L keys for a dense unit), walked in 8-row
// boxes; 16 boxes form a 128-column key tile.  Columns of a box past the end of
// its cluster are masked, so a cluster wastes at most 7 columns.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3 / 4-7  softmax + epilogue of query tile 0 / 1; thread t owns
//                    query row t = TMEM lane t
//   warp 8           TMA producer: Q tiles once; per key tile the K and V
//                    boxes and the tile's column-validity masks
//   warp 9           TMEM allocator and the single-thread tcgen05.mma issuer
//   warps 10-11      idle
// Registers: launched at 168 per thread (65536 / 384, rounded down to 8); the
// third warpgroup drops to 72 and the two softmax warpgroups rise to 200:
// 2 * 128 * 200 + 128 * 72 = 60416 <= 384 * 168 = 64512.
// Tensor memory (512 columns): S_0 | S_1 | O_0 | O_1.  The softmax writes P
// (bf16) over the first half of its S columns and the PV product reads A = P
// from tensor memory, so S, P and O never touch shared memory.  O accumulates
// in TMEM across key tiles; its rows are rescaled only when the running row
// maximum grows by more than 8 (log2 units), so P <= 2^8 stays exact in fp32
// sums and representable in bf16.
// MMA order per key tile j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): while one
// softmax warpgroup works on its S, the tensor core runs the other's products.
// The issuing thread shares its SM sub-partition with two softmax warps, so
// it spends as few instructions per product as it can: descriptors are formed
// once and each group of eight products is one asm block.
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
constexpr int NTHREADS = 384;
constexpr uint32_t kRegsSoftmax = 200, kRegsOther = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= NTHREADS * 168, "register split exceeds the launch");
constexpr float kRescaleLog2 = 8.0f;
constexpr int RG_CACHE = 2048;  // key ranges kept in shared memory (more: read from global)
constexpr int kPolyChunk = 3;   // of the 4 32-column chunks of a key tile, this one takes exp2_poly
// K/V tile layout in shared memory: 16 boxes, each [column half][8 rows][128 B]
// (one 3-D TMA copy per box); an 8-row group is BOX_BYTES after the previous.

template <int D>
struct Layout {
    static constexpr int HALVES = D / 64;  // 128-byte (64 x bf16) column halves
    static constexpr uint32_t Q_TILE = HALVES * BM * 128;
    static constexpr uint32_t KV_BYTES = HALVES * BN * 128;
    static constexpr uint32_t BOX_BYTES = HALVES * 1024;
    static constexpr uint32_t OFF_Q = 0;                        // two query tiles
    static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_TILE;
    static constexpr uint32_t OFF_V = OFF_K + NS * KV_BYTES;
    static constexpr uint32_t OFF_MASK = OFF_V + NS * KV_BYTES;  // [4][4] uint32 (tile j in slot j % 4)
    static constexpr uint32_t OFF_RG = OFF_MASK + 64;            // [RG_CACHE] int2 key ranges
    static constexpr uint32_t OFF_RB = OFF_RG + RG_CACHE * 8;    // [RG_CACHE + 1] first box of each range
    static constexpr uint32_t OFF_CB = OFF_RB + (RG_CACHE + 1) * 4 + 12;  // [4][128] column addends (compensation)
    static constexpr uint32_t OFF_CT = OFF_CB + 4 * BN * 4;      // [4] tile holds centroid columns
    static constexpr uint32_t OFF_BAR = OFF_CT + 16;
    static constexpr uint32_t BYTES = OFF_BAR + 256;
    static constexpr uint32_t SMEM = BYTES + 1024;  // 1024-byte alignment slack
};

enum {
    B_KF = 0,    // [NS] K stage filled (TMA tx) -- also publishes the tile's masks
    B_KE = 2,    // [NS] K stage free (MMA commit after both S products)
    B_VF = 4,    // [NS] V stage filled
    B_VE = 6,    // [NS] V stage free (MMA commit after both PV products)
    B_QF = 8,    // query tiles filled
    B_SF = 9,    // [2] S_i written (MMA commit)
    B_PF = 11,   // [2] P_i written (+ O_i rescaled) by the 128 softmax threads
    B_OF = 13,   // [2] last PV_i complete (MMA commit)
    B_DONE = 15, // every MMA complete
    NBAR = 16
};

// 2^x on the FMA pipe, so that part of the exponentials bypass the
// special-function unit (one ex2 per element would take as long as the two
// matrix products of a tile).  Range reduction x = n + f with n = round(x),
// |f| <= 1/2 (Cody and Waite), n read from the low mantissa bits of
// x + 1.5 * 2^23; 2^f by a cubic fitted here for least maximum relative error
// on [-1/2, 1/2] (1.02e-4, below the 2^-9 rounding of the bf16 P it feeds);
// 2^n added to the exponent field.  x is clamped at -126, so -inf (a masked
// column) gives at most 2^-126 instead of 0.  Two elements per call, in
// packed fp32 pairs.
constexpr float kExp2C3 = 0.05500858277f, kExp2C2 = 0.24221037328f, kExp2C1 = 0.69328290224f;
constexpr float kRoundMagic = 12582912.f;  // 1.5 * 2^23
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float &p0, float &p1) {
    const uint64_t x = f2_pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const uint64_t t = f2_add(x, f2_pack(kRoundMagic, kRoundMagic));
    const uint64_t f = f2_sub(x, f2_sub(t, f2_pack(kRoundMagic, kRoundMagic)));
    uint64_t q = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
    q = f2_fma(q, f, f2_pack(kExp2C1, kExp2C1));
    q = f2_fma(q, f, f2_pack(1.f, 1.f));
    float q0, q1, t0, t1;
    f2_unpack(q, q0, q1);
    f2_unpack(t, t0, t1);
    p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

struct AttnMaps {
    CUtensorMap q;
    CUtensorMap k[4], v[4];  // boxes of 1, 2, 4, 8 row groups
};

struct AttnParams {
    bf16 *O;
    const int *perm_q, *offs_q, *counts_q, *tile_prefix, *nboxes, *nrange, *rbox;
    const int2 *ranges;  // (first 8-row group in Kp / Vp, keys)
    // centroid compensation: index of the range over the centroid rows (-1: none)
    // and, per centroid column, ln|c| / scale, or -inf for a selected or empty cluster
    const int *crange;
    const float *cbias;
    int L, Lpad, Cq, Ccap, BH;
    float scale_log2;
    uint32_t *err;
    unsigned long long *counters;
};

__device__ __forceinline__ void record_wait_failure(const AttnParams &p, int role, int bidx, int j, int par) {
    set_err(p.err, DEV_ERR_TIMEOUT);
    if (p.counters) {
        const unsigned long long code =
            1ull << 60 | (unsigned long long)role << 24 | (unsigned long long)bidx << 16 |
            (unsigned long long)(j & 0x7FFF) << 1 | (unsigned long long)(par & 1);
        atomicCAS(&p.counters[4], 0ull, code);
    }
}

template <int D, bool COMP>
__global__ void __launch_bounds__(NTHREADS, 1)
    k_sparse_attn(const __grid_constant__ AttnMaps maps, const AttnParams p) {
    using LY = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- work item: (unit h, query cluster qc, pair of 128-row tiles)
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
    const int pair = item - p.tile_prefix[hq];
    const int row0 = p.offs_q[(int64_t)h * (p.Cq + 1) + qc] + pair * 2 * BM;
    const int rest = p.counts_q[hq] - pair * 2 * BM;
    const int valid0 = min(BM, rest), valid1 = min(BM, rest - BM);
    const bool has1 = valid1 > 0;
    const int64_t unit_row = (int64_t)h * p.L;
    const int n_tiles = (p.nboxes[hq] + BOXES - 1) / BOXES;
    const int2 *rg = p.ranges + (int64_t)hq * p.Ccap;
    const int *rb = p.rbox + (int64_t)hq * (p.Ccap + 1);
    const int nr = p.nrange[hq];
    const int nbox = p.nboxes[hq];

    const uint32_t bar0 = sbase + LY::OFF_BAR;
#define BAR(i) (bar0 + 8u * (uint32_t)(i))
    // Bounded wait; the first wait to give up anywhere records
    // (role << 24 | barrier << 16 | tile << 1 | parity) in counters[4].
#define WAIT(role, bidx, jj, par)                                                                     \
    (mbar_wait_or_abort(BAR(bidx), (par), p.err) ||                                                   \
     (record_wait_failure(p, (role), (bidx), (jj), (par)), false))
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + LY::OFF_BAR + 8 * NBAR);
    uint32_t *masks = reinterpret_cast<uint32_t *>(sm + LY::OFF_MASK);
    float *cbias_s = reinterpret_cast<float *>(sm + LY::OFF_CB);
    uint32_t *ctile = reinterpret_cast<uint32_t *>(sm + LY::OFF_CT);
    const int cr = COMP ? p.crange[hq] : -1;

    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(BAR(B_KF + i), 1);
            mbar_init(BAR(B_KE + i), 1);
            mbar_init(BAR(B_VF + i), 1);
            mbar_init(BAR(B_VE + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(BAR(B_SF + i), 1);
            mbar_init(BAR(B_PF + i), BM);
            mbar_init(BAR(B_OF + i), 1);
        }
        mbar_init(BAR(B_QF), 1);
        mbar_init(BAR(B_DONE), 1);
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp >= 8) {
      reg_dealloc<kRegsOther>();
      if (warp == 8) {
        // ------------------------------------------------ TMA producer (whole warp)
        // Key tile j is 8-row groups 16j .. 16j+15 of the concatenated walked
        // ranges (every range starts on a group of the padded Kp / Vp).  At
        // most 16 ranges meet a tile: lane l takes the part of range r0 + l
        // inside it, sets its groups' column masks and copies them with as
        // few boxes as possible (8, 4, 2, 1 groups); lanes 16-31 fill the
        // slots past the last group from an all-zero group.
        int2 *rg_s = reinterpret_cast<int2 *>(sm + LY::OFF_RG);
        int *rb_s = reinterpret_cast<int *>(sm + LY::OFF_RB);
        const bool cached = nr <= RG_CACHE;
        if (cached) {
            for (int i = lane; i < nr; i += 32) rg_s[i] = rg[i];
            for (int i = lane; i <= nr; i += 32) rb_s[i] = rb[i];
        }
        __syncwarp();
        const int2 *rgp = cached ? rg_s : rg;
        const int *rbp = cached ? rb_s : rb;
        const int unit_group = h * (p.Lpad / 8);
        const int zero_group = unit_group + p.Lpad / 8 - 1;  // never written: zero
        if (lane == 0) {
            mbar_arrive_expect_tx(BAR(B_QF), 2 * LY::Q_TILE);
            for (int t = 0; t < 2; ++t)
                for (int hf = 0; hf < LY::HALVES; ++hf)
                    tma_load_2d(sbase + LY::OFF_Q + t * LY::Q_TILE + hf * BM * 128, &maps.q, hf * 64,
                                (int)(unit_row + row0 + t * BM), BAR(B_QF));
        }
        int r0 = 0, issued = 0;
        for (int j = 0; j < n_tiles; ++j) {
            const int s = j % NS;
            const int t0 = j * BOXES, t1 = t0 + BOXES;
            const int r = r0 + lane;
            const int rb0 = r <= nr ? rbp[r] : 0x7FFFFFFF;
            const int rb1 = __shfl_down_sync(0xFFFFFFFFu, rb0, 1);
            const bool mine = lane < BOXES && r < nr && rb0 < t1;
            const int a0 = mine ? max(rb0, t0) : 0, a1 = mine ? min(rb1, t1) : 0;
            int2 g = make_int2(0, 0);
            if (mine) g = rgp[r];
            // column masks of the 16 groups (8 bits each, 4 per word) from the
            // groups of this lane's part; the last group of a range may be partial
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t word = 0u;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const int sl = t0 + 4 * q + b;
                    const int v = min(8, g.y - 8 * (sl - rb0));
                    const uint32_t byte = v >= 8 ? 0xFFu : ((1u << max(v, 0)) - 1u);
                    word |= (sl >= a0 && sl < a1) ? byte << (8 * b) : 0u;
                }
                w[q] = __reduce_or_sync(0xFFFFFFFFu, word);
            }
            const int rnext = r0 + __popc(__ballot_sync(0xFFFFFFFFu, mine && rb1 <= t1));
            const int filled = min(max(nbox - t0, 0), BOXES);
            const int gfirst = unit_group + g.x + (a0 - rb0);
            // K: its stage frees once both S products of tile j - NS are done;
            // the masks go to slot j % 4 (the softmax of tile j - 4 is over by then)
            if (j >= NS && !__all_sync(0xFFFFFFFFu, WAIT(1, B_KE + s, j, ((j / NS) - 1) & 1))) {
                ok = false;
                break;
            }
            if (lane < 4) masks[4 * (j & 3) + lane] = lane == 0 ? w[0] : lane == 1 ? w[1] : lane == 2 ? w[2] : w[3];
            if (COMP) {
                // centroid columns of this tile: the addend ln|c| / scale (-inf
                // for the selected and the empty clusters), 0 elsewhere
                const bool cpart = mine && r == cr;
                const bool anyc = __any_sync(0xFFFFFFFFu, cpart);
                if (anyc) {
                    float *cb = cbias_s + (j & 3) * BN;
                    for (int i = lane; i < BN; i += 32) cb[i] = 0.f;
                    __syncwarp();
                    if (cpart) {
                        const float *src = p.cbias + (int64_t)hq * p.Ccap;
                        for (int sl = a0; sl < a1; ++sl)
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int ci = 8 * (sl - rb0) + i;
                                cb[(sl - t0) * 8 + i] = ci < g.y ? src[ci] : 0.f;
                            }
                    }
                }
                if (lane == 0) ctile[j & 3] = anyc ? 1u : 0u;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(BAR(B_KF + s), LY::KV_BYTES);  // releases the masks
            __syncwarp();
            const uint32_t kd = sbase + LY::OFF_K + s * LY::KV_BYTES;
            if (mine) {
                int ls = a0 - t0, gi = gfirst, left = a1 - a0;
                while (left > 0) {
                    const int lg = left >= 8 ? 3 : left >= 4 ? 2 : left >= 2 ? 1 : 0;
                    tma_load_4d(kd + ls * LY::BOX_BYTES, &maps.k[lg], 0, 0, 0, gi, BAR(B_KF + s));
                    ls += 1 << lg;
                    gi += 1 << lg;
                    left -= 1 << lg;
                }
            }
            if (lane >= BOXES && lane - BOXES < BOXES - filled)
                tma_load_4d(kd + (filled + lane - BOXES) * LY::BOX_BYTES, &maps.k[0], 0, 0, 0, zero_group,
                            BAR(B_KF + s));
            // V: its stage frees once both PV products of tile j - NS are done
            if (j >= NS && !__all_sync(0xFFFFFFFFu, WAIT(1, B_VE + s, j, ((j / NS) - 1) & 1))) {
                ok = false;
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(BAR(B_VF + s), LY::KV_BYTES);
            __syncwarp();
            const uint32_t vd = sbase + LY::OFF_V + s * LY::KV_BYTES;
            if (mine) {
                int ls = a0 - t0, gi = gfirst, left = a1 - a0;
                while (left > 0) {
                    const int lg = left >= 8 ? 3 : left >= 4 ? 2 : left >= 2 ? 1 : 0;
                    tma_load_4d(vd + ls * LY::BOX_BYTES, &maps.v[lg], 0, 0, 0, gi, BAR(B_VF + s));
                    ls += 1 << lg;
                    gi += 1 << lg;
                    left -= 1 << lg;
                }
            }
            if (lane >= BOXES && lane - BOXES < BOXES - filled)
                tma_load_4d(vd + (filled + lane - BOXES) * LY::BOX_BYTES, &maps.v[0], 0, 0, 0, zero_group,
                            BAR(B_VF + s));
            r0 = rnext;
            ++issued;
        }
        if (lane == 0) {
            // Loads still in flight must land before the CTA exits.
            for (int j = issued - NS < 0 ? 0 : issued - NS; j < issued; ++j)
                if (!WAIT(2, B_KF + (j % NS), j, (j / NS) & 1) || !WAIT(2, B_VF + (j % NS), j, (j / NS) & 1))
                    ok = false;
            if (!WAIT(2, B_QF, 0, 0)) ok = false;
            if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
        }
        __syncwarp();
      } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IQK = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t IPV = idesc_bf16_f32(BM, D, true);
            // Descriptors are formed once; a product's descriptor is its base
            // plus the operand's offset in 16-byte units (the address field
            // cannot carry: every offset stays inside shared memory).
            const uint64_t dq0 = sdesc_sw128(sbase + LY::OFF_Q, 16, 1024);
            const uint64_t dk0 = sdesc_sw128(sbase + LY::OFF_K, 16, LY::BOX_BYTES);
            const uint64_t dv0 = sdesc_sw128(sbase + LY::OFF_V, 1024, LY::BOX_BYTES);
            auto issue_s = [&](int i, int j) {
                const uint64_t dq = dq0 + (uint64_t)((i * LY::Q_TILE) >> 4);
                const uint64_t dk = dk0 + (uint64_t)(((j % NS) * LY::KV_BYTES) >> 4);
                // K16 step kk reads Q at (kk / 4) x BM x 128 B (its column half) plus
                // (kk % 4) x 32 B and K at (kk / 4) x 1024 B plus (kk % 4) x 32 B; the
                // template arguments are these offsets in 16-byte units
                if constexpr (D == 128) {
                    constexpr uint32_t QH = (BM * 128) >> 4;
                    mma8_ss<2, 4, 6, QH, QH + 2, QH + 4, QH + 6, 2, 4, 6, 64, 66, 68, 70>(tmem + i * BN, dq, dk, IQK, 0u);
                } else {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        tc_mma_bf16(tmem + i * BN, dq + (uint64_t)(kk * 2), dk + (uint64_t)(kk * 2), IQK, kk > 0 ? 1u : 0u);
                }
                tc_commit(BAR(B_SF + i));
            };
            auto issue_pv = [&](int i, int j) {
                const uint64_t dv = dv0 + (uint64_t)(((j % NS) * LY::KV_BYTES) >> 4);
                constexpr uint32_t VSTEP = (2 * LY::BOX_BYTES) / 16;
                mma8_ts<VSTEP>(tmem + 256 + i * 128, tmem + i * BN, dv, IPV, j > 0 ? 1u : 0u);
            };
            if (!WAIT(3, B_QF, 0, 0)) ok = false;
            if (ok && n_tiles > 0) {
                if (!WAIT(3, B_KF, 0, 0)) ok = false;
                tc_fence_after();
                if (ok) {
                    issue_s(0, 0);
                    if (has1) issue_s(1, 0);
                    tc_commit(BAR(B_KE + 0));
                }
            }
            for (int j = 0; j < n_tiles && ok; ++j) {
                const bool more = j + 1 < n_tiles;
                if (!WAIT(3, B_PF + 0, j, j & 1) || !WAIT(3, B_VF + (j % NS), j, (j / NS) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_pv(0, j);
                if (!more) tc_commit(BAR(B_OF + 0));
                if (more) {
                    if (!WAIT(3, B_KF + ((j + 1) % NS), j + 1, ((j + 1) / NS) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_s(0, j + 1);
                }
                if (has1) {
                    if (!WAIT(3, B_PF + 1, j, j & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    issue_pv(1, j);
                    if (!more) tc_commit(BAR(B_OF + 1));
                    if (more) issue_s(1, j + 1);
                }
                if (more) tc_commit(BAR(B_KE + ((j + 1) % NS)));  // K(j+1): both S products issued
                tc_commit(BAR(B_VE + (j % NS)));                  // V(j): both PV products issued
            }
            tc_commit(BAR(B_DONE));
            if (!WAIT(4, B_DONE, 0, 0)) ok = false;
            if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
        }
        __syncwarp();
      }
    } else {
        reg_alloc<kRegsSoftmax>();
        // ------------------------------------------------ softmax + epilogue
        const int wg = warp >> 2;  // query tile
        const int row = tid & 127;
        const int valid = wg == 0 ? valid0 : valid1;
        if (wg == 0 || has1) {
            const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
            const uint32_t tS = tmem + lane_off + wg * BN;
            const uint32_t tO = tmem + lane_off + 256 + wg * 128;
            const float sl2 = p.scale_log2;
            float m_run = -INFINITY, l_run = 0.f;
            long long kept_cols = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int s = j % NS;
                // Wait outcomes are combined across the warp: the TMEM loads and
                // stores below are warp-collective, so a warp leaves together.
                if (!__all_sync(0xFFFFFFFFu, WAIT(5 + wg, B_KF + s, j, (j / NS) & 1))) {
                    ok = false;
                    break;
                }
                const uint4 mk = *reinterpret_cast<const uint4 *>(masks + 4 * (j & 3));
                const uint32_t vm[4] = {mk.x, mk.y, mk.z, mk.w};
                kept_cols += __popc(vm[0]) + __popc(vm[1]) + __popc(vm[2]) + __popc(vm[3]);
                if (!__all_sync(0xFFFFFFFFu, WAIT(5 + wg, B_SF + wg, j, j & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, r[c]);
                tmem_ld_wait();
                // Masked columns become -inf (the masks are the same for every
                // row, so the branch is warp-uniform; most chunks are full).
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (vm[c] != 0xFFFFFFFFu) {
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[c][i] = ((vm[c] >> i) & 1u) ? r[c][i] : 0xFF800000u;
                    }
                }
                if (COMP && ctile[j & 3]) {
                    // a centroid column c stands for |c| keys at its member mean:
                    // its score gains ln|c| / scale (the softmax weight |c| exp(q.k / sqrt d))
                    const float4 *cb = reinterpret_cast<const float4 *>(cbias_s + (j & 3) * BN);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            const float4 b = cb[c * 8 + i / 4];
                            r[c][i] = __float_as_uint(__uint_as_float(r[c][i]) + b.x);
                            r[c][i + 1] = __float_as_uint(__uint_as_float(r[c][i + 1]) + b.y);
                            r[c][i + 2] = __float_as_uint(__uint_as_float(r[c][i + 2]) + b.z);
                            r[c][i + 3] = __float_as_uint(__uint_as_float(r[c][i + 3]) + b.w);
                        }
                }
                // Row maximum: 8 independent partial maxima, three-input max.
                float pm[8];
#pragma unroll
                for (int a = 0; a < 8; ++a) pm[a] = -INFINITY;
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        pm[(i >> 1) & 7] = fmax3(pm[(i >> 1) & 7], __uint_as_float(r[c][i]),
                                                 __uint_as_float(r[c][i + 1]));
                const float tmax = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
                const float m_new = fmaxf(m_run, tmax * sl2);
                // The rescale touches TMEM with warp-collective (.sync.aligned)
                // loads and stores, so the decision must be uniform across the
                // warp: if any row's maximum grew by more than 2^8, every row of
                // the warp moves to its new maximum (factor 1 where it did not grow).
                if (__any_sync(0xFFFFFFFFu, j == 0 || m_new > m_run + kRescaleLog2)) {
                    if (j > 0) {
                        // O_i and l are rescaled to the new maximum (PV_i(j-1) is
                        // complete: S_i(j) was issued after it).
                        const float alpha = m_new > m_run ? ex2_approx(m_run - m_new) : 1.f;
                        l_run *= alpha;
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tO + c * 32, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                            tmem_st32(tO + c * 32, o);
                        }
                        tmem_st_wait();
                    }
                    m_run = m_new;
                }
                // p = 2^(s * scale * log2(e) - m): one FMA and one ex2 per element,
                // in packed pairs; -inf columns give 0.  Row sum with 8
                // independent partial sums (4 packed pairs).
                const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m_run, -m_run);
                uint64_t ps2[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) ps2[a] = f2_pack(0.f, 0.f);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[32];
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c = half * 2 + cc;
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1])),
                                                       sl2x2, negm2);
                            float x0, x1, p0, p1;
                            f2_unpack(x2, x0, x1);
                            if (c == kPolyChunk) {
                                exp2_poly2(x0, x1, p0, p1);
                            } else {
                                p0 = ex2_approx(x0);
                                p1 = ex2_approx(x1);
                            }
                            ps2[(i >> 1) & 3] = f2_add(ps2[(i >> 1) & 3], f2_pack(p0, p1));
                            pk[cc * 16 + (i >> 1)] = pack_bf16x2(p0, p1);
                        }
                    }
                    tmem_st32(tS + half * 32, pk);  // P columns [32*half, 32*half+32)
                }
                float ps[8];
#pragma unroll
                for (int a = 0; a < 4; ++a) f2_unpack(ps2[a], ps[2 * a], ps[2 * a + 1]);
                const float rs = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
                tmem_st_wait();
                l_run += rs;
                tc_fence_before();
                mbar_arrive(BAR(B_PF + wg));
            }
            if (ok && n_tiles > 0) {
                if (!__all_sync(0xFFFFFFFFu, WAIT(7 + wg, B_OF + wg, n_tiles, 0))) ok = false;
            }
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) {
                set_err(p.err, DEV_ERR_TIMEOUT);
            } else {
                tc_fence_after();
                const float il = n_tiles > 0 ? 1.f / l_run : 0.f;
                const bool store = row < valid;
                const int tok = store ? p.perm_q[unit_row + row0 + wg * BM + row] : 0;
                uint4 *dst = reinterpret_cast<uint4 *>(p.O + (unit_row + tok) * D);
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + c * 32, o);
                    tmem_ld_wait();
                    if (store) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float *f = reinterpret_cast<const float *>(o + 8 * q);
                            dst[c * 4 + q] = make_uint4(pack_bf16x2(f[0] * il, f[1] * il),
                                                        pack_bf16x2(f[2] * il, f[3] * il),
                                                        pack_bf16x2(f[4] * il, f[5] * il),
                                                        pack_bf16x2(f[6] * il, f[7] * il));
                        }
                    }
                }
            }
            if (row == 0 && p.counters) {
                atomicAdd(&p.counters[0], (unsigned long long)((long long)valid * kept_cols));
                atomicAdd(&p.counters[1], (unsigned long long)((long long)BM * BN * n_tiles));
                atomicAdd(&p.counters[2], 1ull);
            }
        }
    }
#undef WAIT
#undef BAR
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

int attn_max_tiles(int L, int Cq, int BH) { return BH * ((L + 2 * BM - 1) / (2 * BM) + Cq); }

cudaError_t launch_sparse_attn(const AttnArgs &a, cudaStream_t s) {
    AttnParams p;
    p.O = a.O;
    p.perm_q = a.perm_q;
    p.offs_q = a.offs_q;
    p.counts_q = a.counts_q;
    p.tile_prefix = a.tile_prefix;
    p.nboxes = a.nboxes;
    p.ranges = a.ranges;
    p.rbox = a.rbox;
    p.nrange = a.nrange;
    p.Lpad = a.Lpad;
    p.L = a.L;
    AttnMaps maps;
    maps.q = *a.tm_q;
    for (int i = 0; i < 4; ++i) {
        maps.k[i] = a.tm_kg[i];
        maps.v[i] = a.tm_vg[i];
    }
    p.Cq = a.Cq;
    p.Ccap = a.Ccap;
    p.BH = a.BH;
    p.scale_log2 = a.scale_log2;
    p.err = a.err;
    p.counters = a.counters;
    p.crange = a.crange;
    p.cbias = a.cbias;
    const int grid = attn_max_tiles(a.L, a.Cq, a.BH);
    const bool comp = a.crange != nullptr;
    cudaError_t e;
    auto go = [&](auto kern, uint32_t smem) -> cudaError_t {
        cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        kern<<<grid, NTHREADS, smem, s>>>(maps, p);
        AC_NOTE_LAUNCH();
        return cudaSuccess;
    };
    if (a.d == 128)
        e = comp ? go(k_sparse_attn<128, true>, Layout<128>::SMEM) : go(k_sparse_attn<128, false>, Layout<128>::SMEM);
    else
        e = comp ? go(k_sparse_attn<64, true>, Layout<64>::SMEM) : go(k_sparse_attn<64, false>, Layout<64>::SMEM);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace ac
