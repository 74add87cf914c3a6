// assign_mma.cu -- k-means assignment on tcgen05 tensor cores with exact
// decisions (AdaCluster, arXiv 2604.18348: Sec. 3.1 angular k-means of the
// queries; Sec. 3.2.2, Algorithm 1 and the warm-started k-means of the keys).
//
// The label of a row x is argmin_c D(x, c), D the fp32 squared distance summed
// in dimension order, ties to the lowest c.  Evaluating every D that way costs
// three dependent fp32 operations per (row, centre, dimension) on CUDA cores.
// Here instead:
//   1. each centre is represented as c' = c_hi (+ c_lo) with c_hi = bf16(c)
//      (and c_lo = bf16(c - c_hi) where the pass asks for two terms); the
//      tensor cores form s = x . c' for every centre (key rows are exact bf16;
//      query rows are scaled by their fp32 inverse norm afterwards);
//   2. the epilogue keeps per row the 4 smallest A(c) = |c'|^2 - 2 s, the
//      squared distance to c' less the row's own |x|^2 (for keys the tensor
//      cores add |c'|^2 too: the centre rows hold -2 c_hi, and one more K=16
//      slice multiplies a constant [1 1 1 0 ...] row by |c'|^2 split into three
//      bf16 parts, so the accumulator holds A itself);
//   3. a rigorous bound E on |D(x, c) - |x|^2 - A(c)| (bf16 split, tensor-core
//      accumulation, the fp32 rounding of D itself; see assign_bound) decides:
//      when every other centre's lower bound A - E lies above the best's upper
//      bound, the best is the exact argmin; otherwise the row's candidates (or,
//      rarely, all centres) are rescored with the exact arithmetic.
// The labels are therefore those of the exact definition.  dmin, where used,
// is recomputed exactly for the chosen centre.
#include "ac_device.cuh"
#include "ac_internal.h"

namespace ac {
namespace {

constexpr int AM = 128;       // rows per MMA (M)
constexpr int AU = 2 * AM;    // rows per work unit: two MMAs share every centre chunk
constexpr int ACH = 128;      // centres per chunk at most (MMA N)
constexpr int A_EPI = 256;    // epilogue threads: one per row of the unit
constexpr int A_THREADS = A_EPI + 64;
constexpr int A_NC = 2;       // centre chunk stages
constexpr int QCH = 96;       // query centres per chunk at most (c_hi and c_lo: twice the operand bytes)
constexpr int A_NCMAX = 3;    // barriers reserved

// Shared memory: [2] row units (two 128-row tiles each) | [NC] centre chunks.
// A chunk holds the c_hi rows (and the c_lo rows) of up to ACH centres, each
// operand as [column half][rows][128 B] with the 128-byte swizzle.
template <int D, bool FOLD>
struct ALayout {
    static constexpr int HALVES = D / 64;
    static constexpr uint32_t XT_BYTES = HALVES * AM * 128;  // one 128-row tile
    static constexpr uint32_t X_BYTES = 2 * XT_BYTES;        // one unit
    static constexpr uint32_t OFF_X = 0;
    static constexpr uint32_t OFF_C = OFF_X + 2 * X_BYTES;
    // two stages of ACH key centres (-2 c_hi, then the |c'|^2 slice: two
    // no-swizzle 16-byte columns of ACH rows), or of up to QCH query centres
    // (c_hi, c_lo)
    static constexpr uint32_t C_REGION =
        FOLD ? A_NC * (HALVES * ACH * 128 + ACH * 32) : A_NC * (2 * HALVES * QCH * 128);
    static constexpr uint32_t OFF_XE = OFF_C + C_REGION;  // keys: the constant [1 1 1 0 ...] K slice, 128 rows
    static constexpr uint32_t OFF_BAR = OFF_XE + (FOLD ? AM * 32 : 0);
    static constexpr uint32_t BYTES = OFF_BAR + 256;
    static constexpr uint32_t SMEM = BYTES + 1024;
};

// barriers
enum {
    B_XF = 0,    // [2] row unit landed
    B_XE = 2,    // [2] row unit consumed by the MMAs
    B_CF = 4,    // [3] centre chunk landed
    B_CE = 7,    // [3] centre chunk consumed
    B_AF = 10,   // [2] accumulators of a chunk ready
    B_AE = 12,   // [2] accumulators drained (256 arrivals)
    B_DONE = 14,
    B_N = 15
};

struct AsgParams {
    const float *inv;     // [BH, L] (queries) or null
    const float *rowsq;   // [BH, L] |x|^2 (keys) or null (normalised rows: 1)
    const float *cn;      // [BH, Cpad]
    const unsigned int *hstat;  // [BH, 2] max delta, max |c_hi|^2 (float bits)
    const int *nrows; int nrows_const;
    const int *ncent; int ncent_const;
    int64_t L;
    int BH, Cpad, CH, units_per_head;
    int two_term;         // c' = c_hi + c_lo (else c_hi)
    int nc;               // centre chunk stages
    uint32_t c_stage;     // bytes of one centre chunk stage
    float e_tc;           // tensor-core error coefficient (see assign_bound)
    int *labels;
    int4 *cand;
    int *amb_list, *amb_count;  // candidate rows from the front, every-centre rows from the back
    int64_t amb_cap;            // entries of amb_list
    unsigned long long *stats;  // [0] ambiguous rows, [1] rows rescored against every centre
    uint32_t *err;
};

// Upper bound of |D(x, c) - |x|^2 - A(c)| for a centre with A(c) = a.
//   dup   = max(a + |x|^2, 0) + 2 e  bounds |x - c'|^2 (e covers the error
//           of a: the tensor core's fp32 accumulation of the n products --
//           allowed two units in the last place per addition, twice the
//           round-to-nearest bound, so n 2^-23 (|x|^2 + |c'|^2) --, the query
//           scaling and the roundings of |c'|^2 and of a);
//   |x - c|^2 - |x - c'|^2 is at most 2 sqrt(dup) delta + delta^2 (triangle
//   inequality, delta = max |c - c'|);
//   D itself, d products and d - 1 sums in fp32, is within (d + 2) 2^-24 of
//   |x - c|^2 <= (sqrt(dup) + delta)^2; 2^-16 covers d <= 128.
// The result is widened by 2^-10 of itself plus 2^-20 of the magnitudes for
// the rounding of this fp32 evaluation and of the comparisons.
__device__ __forceinline__ float assign_bound(float a, float sq, float delta, float e) {
    const float dup = fmaxf(a + sq, 0.f) + 2.f * e;
    const float r = sqrtf(dup);
    const float split = (2.f * r + delta) * delta;
    const float rr = r + delta;
    const float b = split + e + 1.52587890625e-05f * rr * rr + 9.5367431640625e-07f * (fabsf(a) + sq);
    return b * 1.0009765625f;
}

__device__ __forceinline__ void top4_insert(float v, int c, float &d1, float &d2, float &d3, float &d4, int &i1,
                                            int &i2, int &i3, int &i4) {
    if (v < d4) {
        if (v < d3) {
            d4 = d3;
            i4 = i3;
            if (v < d2) {
                d3 = d2;
                i3 = i2;
                if (v < d1) {
                    d2 = d1;
                    i2 = i1;
                    d1 = v;
                    i1 = c;
                } else {
                    d2 = v;
                    i2 = c;
                }
            } else {
                d3 = v;
                i3 = c;
            }
        } else {
            d4 = v;
            i4 = c;
        }
    }
}

// r[i] for a run-time i without local memory: a 5-level select tree.
__device__ __forceinline__ float pick32(const uint32_t (&r)[32], int i) {
    uint32_t a[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) a[k] = (i & 1) ? r[2 * k + 1] : r[2 * k];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = (i & 2) ? a[2 * k + 1] : a[2 * k];
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = (i & 4) ? a[2 * k + 1] : a[2 * k];
#pragma unroll
    for (int k = 0; k < 2; ++k) a[k] = (i & 8) ? a[2 * k + 1] : a[2 * k];
    return __uint_as_float((i & 16) ? a[1] : a[0]);
}

// Largest A that can still matter once the best so far is d1: every centre
// with A > T has A - E(A) > d1 + E(d1) >= the final best's upper bound.  With
// sqrt(dup) > 2 delta the slope of E is below 0.51, so T = d1 + 4.5 E(d1)
// suffices; otherwise A - E(A) need not grow with A and nothing is skipped.
__device__ __forceinline__ float assign_threshold(float d1, float sq, float delta, float e) {
    if (!(d1 < INFINITY)) return INFINITY;
    if (sqrtf(fmaxf(d1 + sq, 0.f) + 2.f * e) <= 2.f * delta) return INFINITY;
    return d1 + 4.5f * assign_bound(d1, sq, delta, e);
}

template <int D, bool FOLD>
__global__ void __launch_bounds__(A_THREADS, 1)
    k_assign_mma(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_c,
                 const __grid_constant__ CUtensorMap tm_cn, const AsgParams p) {
    using LY = ALayout<D, FOLD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t bar0 = sbase + LY::OFF_BAR;
#define ABAR(i) (bar0 + 8u * (uint32_t)(i))
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + LY::OFF_BAR + 8 * B_N);
    const int nc = p.nc;
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(ABAR(B_XF + i), 1);
            mbar_init(ABAR(B_XE + i), 1);
            mbar_init(ABAR(B_AF + i), 1);
            mbar_init(ABAR(B_AE + i), A_EPI);
        }
        for (int i = 0; i < A_NCMAX; ++i) {
            mbar_init(ABAR(B_CF + i), 1);
            mbar_init(ABAR(B_CE + i), 1);
        }
        mbar_init(ABAR(B_DONE), 1);
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    if (FOLD && tid < AM) {
        // K slice of ones against the |c'|^2 parts: row r = [1 1 1 0 0 0 0 0 | 0 ...] as
        // core matrices [8-row group][16-byte column][8 rows][16 B] (SBO 256, LBO 128)
        uint4 *xe = reinterpret_cast<uint4 *>(sm + LY::OFF_XE);
        const int grp = tid >> 3, rr = tid & 7;
        xe[grp * 16 + rr] = make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
        xe[grp * 16 + 8 + rr] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nunits = p.BH * p.units_per_head;
    const uint32_t terms = p.two_term ? 2u : 1u;
    bool ok = true;

    if (warp == 8) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t g = 0, uc = 0;
            for (int t = blockIdx.x; t < nunits && ok; t += gridDim.x) {
                const int h = t / p.units_per_head, ru = t % p.units_per_head;
                const int n = p.nrows ? p.nrows[h] : p.nrows_const;
                const int m = p.ncent ? p.ncent[h] : p.ncent_const;
                if (ru * AU >= n || m <= 0) continue;
                const uint32_t xs = uc & 1;
                if (uc >= 2 && !mbar_wait_or_abort(ABAR(B_XE + xs), ((uc >> 1) - 1) & 1, p.err)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(ABAR(B_XF + xs), LY::X_BYTES);
                for (int i = 0; i < 2; ++i)
                    for (int hf = 0; hf < LY::HALVES; ++hf)
                        tma_load_2d(sbase + LY::OFF_X + xs * LY::X_BYTES + i * LY::XT_BYTES + hf * AM * 128, &tm_x,
                                    hf * 64, (int)(h * p.L + ru * AU + i * AM), ABAR(B_XF + xs));
                ++uc;
                const int nch = (m + p.CH - 1) / p.CH;
                for (int ch = 0; ch < nch; ++ch, ++g) {
                    const uint32_t c = g % nc, k = g / nc;
                    if (g >= (uint32_t)nc && !mbar_wait_or_abort(ABAR(B_CE + c), (k - 1) & 1, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t cs = sbase + LY::OFF_C + c * p.c_stage;
                    mbar_arrive_expect_tx(ABAR(B_CF + c), terms * LY::HALVES * p.CH * 128 + (FOLD ? p.CH * 32 : 0));
                    if (FOLD)  // the |c'|^2 parts: two 8-column boxes of CH rows, no swizzle
                        for (int q = 0; q < 2; ++q)
                            tma_load_2d(cs + LY::HALVES * p.CH * 128 + q * p.CH * 16, &tm_cn, q * 8,
                                        h * p.Cpad + ch * p.CH, ABAR(B_CF + c));
                    for (int hf = 0; hf < LY::HALVES; ++hf)
                        tma_load_2d(cs + hf * p.CH * 128, &tm_c, hf * 64, h * p.Cpad + ch * p.CH, ABAR(B_CF + c));
                    if (p.two_term)  // c_lo rows follow the c_hi rows of all units in the tensor map
                        for (int hf = 0; hf < LY::HALVES; ++hf)
                            tma_load_2d(cs + (LY::HALVES + hf) * p.CH * 128, &tm_c, hf * 64,
                                        (p.BH + h) * p.Cpad + ch * p.CH, ABAR(B_CF + c));
                }
            }
            // nothing may still be landing in shared memory when the block exits
            for (uint32_t k = (g >= (uint32_t)nc ? g - nc : 0); k < g; ++k)
                mbar_wait(ABAR(B_CF + (k % nc)), (k / nc) & 1);
            for (uint32_t k = (uc >= 2 ? uc - 2 : 0); k < uc; ++k) mbar_wait(ABAR(B_XF + (k & 1)), (k >> 1) & 1);
            if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t g = 0, uc = 0;
            for (int t = blockIdx.x; t < nunits && ok; t += gridDim.x) {
                const int h = t / p.units_per_head, ru = t % p.units_per_head;
                const int n = p.nrows ? p.nrows[h] : p.nrows_const;
                const int m = p.ncent ? p.ncent[h] : p.ncent_const;
                if (ru * AU >= n || m <= 0) continue;
                const uint32_t xs = uc & 1;
                if (!mbar_wait_or_abort(ABAR(B_XF + xs), (uc >> 1) & 1, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t xa = sbase + LY::OFF_X + xs * LY::X_BYTES;
                const int nch = (m + p.CH - 1) / p.CH;
                for (int ch = 0; ch < nch; ++ch, ++g) {
                    const uint32_t c = g % nc, a = g & 1;
                    if (!mbar_wait_or_abort(ABAR(B_CF + c), (g / nc) & 1, p.err) ||
                        (g >= 2 && !mbar_wait_or_abort(ABAR(B_AE + a), ((g >> 1) - 1) & 1, p.err))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int rem = m - ch * p.CH;
                    const int N = rem >= p.CH ? p.CH : ((rem + 31) & ~31);
                    const uint32_t idesc = idesc_bf16_f32(AM, N, false);
                    const uint32_t ca = sbase + LY::OFF_C + c * p.c_stage;
                    const int nk = (int)terms * (D / 16);
                    for (int i = 0; i < 2; ++i) {
                        for (int kk = 0; kk < nk; ++kk) {
                            const int kx = kk % (D / 16);  // x . c_hi, then x . c_lo
                            const uint32_t xoff = i * LY::XT_BYTES + (kx >> 2) * (AM * 128) + (kx & 3) * 32;
                            const uint32_t coff = (kk >> 2) * (p.CH * 128) + (kk & 3) * 32;
                            tc_mma_bf16(tmem + (a * 2 + i) * ACH, sdesc_sw128(xa + xoff, 16, 1024),
                                        sdesc_sw128(ca + coff, 16, 1024), idesc, kk > 0 ? 1u : 0u);
                        }
                        if (FOLD)  // + |c'|^2 (ones x parts)
                            tc_mma_bf16(tmem + (a * 2 + i) * ACH, sdesc_noswz(sbase + LY::OFF_XE, 128, 256),
                                        sdesc_noswz(ca + LY::HALVES * p.CH * 128, p.CH * 16, 128), idesc, 1u);
                    }
                    tc_commit(ABAR(B_AF + a));
                    tc_commit(ABAR(B_CE + c));
                }
                if (!ok) break;
                tc_commit(ABAR(B_XE + xs));
                ++uc;
            }
            tc_commit(ABAR(B_DONE));
            if (!mbar_wait(ABAR(B_DONE), 0)) ok = false;
            if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        // Warp w owns rows 32 (w % 4) .. + 31 of tile w / 4 of the unit (tensor
        // memory lanes 32 (w % 4) ..), one row per thread, all centres.  A
        // 32-column group costs one FMA and one min per centre; only groups
        // whose minimum reaches the threshold T of assign_threshold (rare after
        // the first ones) mark their columns under it and insert those into the
        // row's top-4 list.  The per-row and per-unit scalars of the next unit
        // and the centre norms of the next group are loaded ahead.
        const int ti = warp >> 2;
        const int rloc = ti * AM + (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        struct UnitScalars {
            float inv, sq;
            uint32_t delta, cmax;
            int m;
        };
        auto fetch = [&](int tt, UnitScalars &v) {
            if (tt >= nunits) return;
            const int hh = tt / p.units_per_head;
            const int row = (tt % p.units_per_head) * AU + rloc;
            const int nn = p.nrows ? p.nrows[hh] : p.nrows_const;
            const int64_t ff = (int64_t)hh * p.L + row;
            v.m = p.ncent ? p.ncent[hh] : p.ncent_const;
            v.inv = p.inv && row < nn ? p.inv[ff] : 1.f;
            v.sq = p.rowsq && row < nn ? p.rowsq[ff] : 1.f;
            v.delta = p.hstat[2 * hh];
            v.cmax = p.hstat[2 * hh + 1];
        };
        auto load_cn = [&](const float *src, float4 (&dst)[8]) {
            const float4 *cn4 = reinterpret_cast<const float4 *>(src);
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = __ldg(cn4 + q);
        };
        UnitScalars cur{1.f, 1.f, 0u, 0u, 0}, nxt{1.f, 1.f, 0u, 0u, 0};
        fetch(blockIdx.x, cur);
        uint32_t g = 0;
        for (int t = blockIdx.x; t < nunits && ok; t += gridDim.x, cur = nxt) {
            fetch(t + gridDim.x, nxt);
            const int h = t / p.units_per_head, ru = t % p.units_per_head;
            const int n = p.nrows ? p.nrows[h] : p.nrows_const;
            const int m = cur.m;
            if (ru * AU >= n || m <= 0) continue;
            const int row = ru * AU + rloc;
            const bool valid = row < n;
            const int64_t f = (int64_t)h * p.L + row;
            const float m2i = -2.f * cur.inv;
            const float sq = cur.sq;
            const float delta = __uint_as_float(cur.delta);
            const float e = p.e_tc * (sq + __uint_as_float(cur.cmax));
            const float *cnh = p.cn + (int64_t)h * p.Cpad;
            float d1 = INFINITY, d2 = INFINITY, d3 = INFINITY, d4 = INFINITY;
            int i1 = 0, i2 = -1, i3 = -1, i4 = -1;
            float T = INFINITY;
            const int nch = (m + p.CH - 1) / p.CH;
            float4 cq[8];
            if (!FOLD) load_cn(cnh, cq);
            for (int ch = 0; ch < nch; ++ch, ++g) {
                const uint32_t a = g & 1;
                const int rem = m - ch * p.CH;
                const int N = rem >= p.CH ? p.CH : ((rem + 31) & ~31);
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_or_abort(ABAR(B_AF + a), (g >> 1) & 1, p.err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (FOLD) {
                    // keys: the whole chunk (up to four 32-column groups) at once;
                    // its minimum sets the threshold before any column is marked,
                    // so only columns near the best of the chunk reach the top-4
                    uint32_t r[4][32];
#pragma unroll
                    for (int g = 0; g < 4; ++g)
                        if (g * 32 < N) tmem_ld32(tmem + lane_off + (a * 2 + ti) * ACH + g * 32, r[g]);
                    tmem_ld_wait();
                    float gm[4];
                    float cm = INFINITY;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float pmn[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
                        if (g * 32 < N) {
#pragma unroll
                            for (int q = 0; q < 16; ++q)
                                pmn[q & 3] = fmin3(pmn[q & 3], __uint_as_float(r[g][2 * q]), __uint_as_float(r[g][2 * q + 1]));
                        }
                        gm[g] = fminf(fmin3(pmn[0], pmn[1], pmn[2]), pmn[3]);
                        cm = fminf(cm, gm[g]);
                    }
                    const bool need = cm <= T;
                    if (__any_sync(0xFFFFFFFFu, need)) {
                        const float Tn = need ? assign_threshold(fminf(d1, cm), sq, delta, e) : T;
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const bool ng = need && g * 32 < N && gm[g] <= Tn;
                            if (__any_sync(0xFFFFFFFFu, ng)) {
                                uint32_t msk = 0u;
#pragma unroll
                                for (int i = 0; i < 32; ++i) msk |= __uint_as_float(r[g][i]) <= Tn ? (1u << i) : 0u;
                                if (ng) {
                                    const int c0 = ch * p.CH + g * 32;
                                    for (uint32_t mm = msk; mm != 0u; mm &= mm - 1u) {
                                        const int i = __ffs(mm) - 1;
                                        top4_insert(pick32(r[g], i), c0 + i, d1, d2, d3, d4, i1, i2, i3, i4);
                                    }
                                }
                            }
                        }
                        if (need) T = Tn;
                    }
                } else
                for (int cg = 0; cg < N; cg += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem + lane_off + (a * 2 + ti) * ACH + cg, r);
                    float4 cqn[8];
                    if (!FOLD) {
                        // norms of the next group: same chunk, else the next chunk
                        const int ncg = cg + 32 < N ? ch * p.CH + cg + 32 : (ch + 1) * p.CH;
                        if (ncg < m) load_cn(cnh + ncg, cqn);
                    }
                    tmem_ld_wait();
                    float mn = INFINITY;
                    if (FOLD) {  // the accumulator holds A already: 4 partial minima, 3-input min
                        float pmn[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
#pragma unroll
                        for (int q = 0; q < 16; ++q)
                            pmn[q & 3] = fmin3(pmn[q & 3], __uint_as_float(r[2 * q]), __uint_as_float(r[2 * q + 1]));
                        mn = fminf(fmin3(pmn[0], pmn[1], pmn[2]), pmn[3]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float v0 = fmaf(m2i, __uint_as_float(r[4 * q + 0]), cq[q].x);
                            const float v1 = fmaf(m2i, __uint_as_float(r[4 * q + 1]), cq[q].y);
                            const float v2 = fmaf(m2i, __uint_as_float(r[4 * q + 2]), cq[q].z);
                            const float v3 = fmaf(m2i, __uint_as_float(r[4 * q + 3]), cq[q].w);
                            r[4 * q + 0] = __float_as_uint(v0);
                            r[4 * q + 1] = __float_as_uint(v1);
                            r[4 * q + 2] = __float_as_uint(v2);
                            r[4 * q + 3] = __float_as_uint(v3);
                            mn = fminf(mn, fminf(fminf(v0, v1), fminf(v2, v3)));
                        }
                    }
                    // This group holds the best so far or a near tie for some
                    // row of the warp: mark the columns within the new threshold
                    // (one compare and one select per column, the same
                    // instructions in every lane), then insert the marked ones.
                    const bool need = mn <= T;
                    if (__any_sync(0xFFFFFFFFu, need)) {
                        const float Tn = need ? assign_threshold(fminf(d1, mn), sq, delta, e) : T;
                        uint32_t msk = 0u;
#pragma unroll
                        for (int i = 0; i < 32; ++i) msk |= __uint_as_float(r[i]) <= Tn ? (1u << i) : 0u;
                        if (need) {
                            T = Tn;
                            const int c0 = ch * p.CH + cg;
                            // the value of column i is picked from the 32
                            // registers by a select tree on i
                            for (uint32_t mm = msk; mm != 0u; mm &= mm - 1u) {
                                const int i = __ffs(mm) - 1;
                                top4_insert(pick32(r, i), c0 + i, d1, d2, d3, d4, i1, i2, i3, i4);
                            }
                        }
                    }
                    if (!FOLD) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) cq[q] = cqn[q];
                    }
                }
                tc_fence_before();
                mbar_arrive(ABAR(B_AE + a));
            }
            if (!ok) break;
            if (valid) {
                const float ub = d1 + assign_bound(d1, sq, delta, e);
                const bool a2 = i2 >= 0 && d2 - assign_bound(d2, sq, delta, e) <= ub;
                const bool a3 = i3 >= 0 && d3 - assign_bound(d3, sq, delta, e) <= ub;
                const bool a4 = i4 >= 0 && d4 - assign_bound(d4, sq, delta, e) <= ub;
                // A - E(A) grows with A once sqrt(dup) > delta, so the centres
                // beyond the kept four are settled when the fourth is.
                const bool beyond = m > 4 && (a4 || sqrtf(fmaxf(d4 + sq, 0.f) + 2.f * e) <= 2.f * delta);
                p.labels[f] = i1;
                if (beyond) {
                    const int pos = atomicAdd(p.amb_count + 1, 1);
                    p.amb_list[p.amb_cap - 1 - pos] = (int)f;
                } else if (a2 || a3 || a4) {
                    const int pos = atomicAdd(p.amb_count, 1);
                    p.amb_list[pos] = (int)f;
                    p.cand[pos] = make_int4(i1, a2 ? i2 : -1, a3 ? i3 : -1, a4 ? i4 : -1);
                }
            }
        }
        if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
    }
#undef ABAR
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Exact fp32 squared distance, dimensions in order (the definition's arithmetic).
// The row and the centre are read 32 dimensions at a time, all loads of a block
// issued before its arithmetic, so the load latency is paid d / 32 times.
template <bool NORM>
__device__ __forceinline__ float exact_sqdist(const bf16 *__restrict__ xr, float s, const float *__restrict__ c,
                                              int d) {
    float acc = 0.f;
    const uint4 *x8 = reinterpret_cast<const uint4 *>(xr);
    const float4 *c4 = reinterpret_cast<const float4 *>(c);
    for (int b = 0; b < d / 32; ++b) {
        uint4 xv[4];
        float4 cv[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = x8[4 * b + q];
#pragma unroll
        for (int q = 0; q < 8; ++q) cv[q] = c4[8 * b + q];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t w[4] = {xv[q].x, xv[q].y, xv[q].z, xv[q].w};
            const float cc[8] = {cv[2 * q].x, cv[2 * q].y, cv[2 * q].z, cv[2 * q].w,
                                 cv[2 * q + 1].x, cv[2 * q + 1].y, cv[2 * q + 1].z, cv[2 * q + 1].w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float x = __uint_as_float((j & 1) ? (w[j >> 1] & 0xFFFF0000u) : (w[j >> 1] << 16));
                if (NORM) x = __fmul_rn(x, s);
                const float t = __fsub_rn(x, cc[j]);
                acc = __fadd_rn(acc, __fmul_rn(t, t));
            }
        }
    }
    return acc;
}

// Rows with a few candidates: four consecutive lanes per row, lane j of the
// group computes the exact distance of candidate j; the group's argmin takes
// the lowest index among equal distances.
template <bool NORM>
__global__ void k_assign_resolve(const bf16 *__restrict__ X, const float *__restrict__ inv, int64_t L, int d,
                                 const float *__restrict__ C, int64_t cstride, const int4 *__restrict__ cand,
                                 const int *__restrict__ amb_list, const int *__restrict__ amb_count,
                                 int *__restrict__ labels, unsigned long long *__restrict__ stats) {
    const int n = amb_count[0];
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        atomicAdd(stats, (unsigned long long)(n + amb_count[1]));
        atomicAdd(stats + 1, (unsigned long long)amb_count[1]);
    }
    const int lane = threadIdx.x & 31, j = lane & 3;
    const int64_t nthr = (int64_t)gridDim.x * blockDim.x;
    // the loop bound is uniform per warp, so every lane takes part in the shuffles
    for (int64_t base = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) - lane; base < 4 * (int64_t)n;
         base += nthr) {
        const int64_t t = base + lane;
        const int i = (int)(t >> 2);
        float best = INFINITY;
        int arg = 0x7FFFFFFF;
        int64_t f = 0;
        if (i < n) {
            f = amb_list[i];
            const int4 cd = cand[i];
            const int c = j == 0 ? cd.x : j == 1 ? cd.y : j == 2 ? cd.z : cd.w;
            if (c >= 0) {
                const int h = (int)(f / L);
                best = exact_sqdist<NORM>(X + f * d, NORM ? inv[f] : 1.f, C + (int64_t)h * cstride + (int64_t)c * d, d);
                arg = c;
            }
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            const float ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
            const int oa = __shfl_xor_sync(0xFFFFFFFFu, arg, o);
            if (ob < best || (ob == best && oa < arg)) {
                best = ob;
                arg = oa;
            }
        }
        if (i < n && j == 0) labels[f] = arg;
    }
}

// Rows whose every centre stays in doubt: one block per row, thread t scores
// centres t, t + blockDim, ... in ascending order; lowest index on ties.
template <bool NORM>
__global__ void k_assign_resolve_all(const bf16 *__restrict__ X, const float *__restrict__ inv, int64_t L, int d,
                                     const float *__restrict__ C, int64_t cstride, const int *__restrict__ ncent,
                                     int ncent_const, const int *__restrict__ amb_list, int64_t amb_cap,
                                     const int *__restrict__ amb_count, int *__restrict__ labels) {
    __shared__ float sb[32];
    __shared__ int sa[32];
    const int n = amb_count[1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        const int64_t f = amb_list[amb_cap - 1 - i];
        const int h = (int)(f / L);
        const int m = ncent ? ncent[h] : ncent_const;
        const bf16 *xr = X + f * d;
        const float s = NORM ? inv[f] : 1.f;
        const float *Ch = C + (int64_t)h * cstride;
        float best = INFINITY;
        int arg = 0x7FFFFFFF;
        for (int c = threadIdx.x; c < m; c += blockDim.x) {
            const float v = exact_sqdist<NORM>(xr, s, Ch + (int64_t)c * d, d);
            if (v < best) {
                best = v;
                arg = c;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xFFFFFFFFu, best, o);
            const int oa = __shfl_xor_sync(0xFFFFFFFFu, arg, o);
            if (ob < best || (ob == best && oa < arg)) {
                best = ob;
                arg = oa;
            }
        }
        if (lane == 0) {
            sb[warp] = best;
            sa[warp] = arg;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            for (int w = 1; w < nwarp; ++w)
                if (sb[w] < best || (sb[w] == best && sa[w] < arg)) {
                    best = sb[w];
                    arg = sa[w];
                }
            labels[f] = arg == 0x7FFFFFFF ? 0 : arg;
        }
        __syncthreads();
    }
}

template <bool NORM>
__global__ void k_exact_dmin(const bf16 *__restrict__ X, const float *__restrict__ inv, int64_t L, int d,
                             const float *__restrict__ C, int64_t cstride, const int *__restrict__ nrows,
                             int nrows_const, const int *__restrict__ ncent, int ncent_const,
                             const int *__restrict__ labels, float *__restrict__ dmin) {
    const int h = blockIdx.y;
    const int row = blockIdx.x * blockDim.x + threadIdx.x;
    const int n = nrows ? nrows[h] : nrows_const;
    const int m = ncent ? ncent[h] : ncent_const;
    if (row >= n || m <= 0) return;
    const int64_t f = (int64_t)h * L + row;
    dmin[f] = exact_sqdist<NORM>(X + f * d, NORM ? inv[f] : 1.f, C + (int64_t)h * cstride + (int64_t)labels[f] * d,
                                 d);
}

// |x|^2 of every row (it only enters the error bound; fp32 is enough).
__global__ void k_row_sqnorm(const bf16 *__restrict__ X, int64_t rows, int d, float *__restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(X + i * d);
    float ss = 0.f;
    for (int k8 = 0; k8 < d / 8; ++k8) {
        const uint4 v = src[k8];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float a = __uint_as_float(w[t] << 16), b = __uint_as_float(w[t] & 0xFFFF0000u);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
        }
    }
    out[i] = ss;
}

// c_hi = bf16(c) (nearest), c_lo = bf16(c - c_hi) with two terms, c' their
// sum; cn = fp32(|c'|^2); per unit the largest delta = |c - c'| and the
// largest |c'|^2, both in fp64 rounded up.  Chi holds [BH, Cpad, d] c_hi rows
// then (two terms) [BH, Cpad, d] c_lo rows.  Rows c >= m up to Cpad are zero
// with cn = +inf.
// With fold (keys), Chi holds -2 c_hi instead (exact: a power-of-two scale) and
// cnp [BH, Cpad, 16] the parts hi, mid, lo of fp32 |c'|^2 as bf16 (their sum is
// |c'|^2 to 2^-26 relative), then zeros; a padding row's first part is the
// largest finite bf16, so its A never wins.
__global__ void k_centre_prep(const float *__restrict__ C, int64_t cstride, const int *__restrict__ ncent,
                              int ncent_const, int d, int Cpad, int two_term, int fold, bf16 *__restrict__ Chi,
                              bf16 *__restrict__ cnp, float *__restrict__ cn, unsigned int *__restrict__ hstat) {
    const int c = blockIdx.x, h = blockIdx.y;
    const int m = ncent ? ncent[h] : ncent_const;
    const int64_t lo_off = (int64_t)gridDim.y * Cpad * d;
    bf16 *dst = Chi + ((int64_t)h * Cpad + c) * d;
    bf16 *pn = fold ? cnp + ((int64_t)h * Cpad + c) * 16 : nullptr;
    if (c >= m) {
        for (int k = threadIdx.x; k < d; k += blockDim.x) {
            dst[k] = __float2bfloat16_rn(0.f);
            if (two_term) dst[lo_off + k] = __float2bfloat16_rn(0.f);
        }
        if (fold && threadIdx.x < 16) pn[threadIdx.x] = __ushort_as_bfloat16(threadIdx.x == 0 ? 0x7F7Fu : 0u);
        if (threadIdx.x == 0) cn[(int64_t)h * Cpad + c] = INFINITY;
        return;
    }
    const float *src = C + (int64_t)h * cstride + (int64_t)c * d;
    double e2 = 0.0, n2 = 0.0;
    for (int k = threadIdx.x; k < d; k += blockDim.x) {
        const float v = src[k];
        const bf16 hi = __float2bfloat16_rn(v);
        dst[k] = fold ? __float2bfloat16_rn(-2.f * __bfloat162float(hi)) : hi;
        double rep = (double)__bfloat162float(hi);
        if (two_term) {
            const bf16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));  // v - hi is exact in fp32
            dst[lo_off + k] = lo;
            rep += (double)__bfloat162float(lo);
        }
        const double r = (double)v - rep;
        e2 += r * r;
        n2 += rep * rep;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        e2 += __shfl_down_sync(0xFFFFFFFFu, e2, o);
        n2 += __shfl_down_sync(0xFFFFFFFFu, n2, o);
    }
    __shared__ double se[4], sn[4];
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        se[w] = e2;
        sn[w] = n2;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double te = 0.0, tn = 0.0;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) {
            te += se[i];
            tn += sn[i];
        }
        const float cnf = (float)tn;
        cn[(int64_t)h * Cpad + c] = cnf;
        if (fold) {
            const bf16 p0 = __float2bfloat16_rn(cnf);
            const float r1 = cnf - __bfloat162float(p0);
            const bf16 p1 = __float2bfloat16_rn(r1);
            const bf16 p2 = __float2bfloat16_rn(r1 - __bfloat162float(p1));
            pn[0] = p0;
            pn[1] = p1;
            pn[2] = p2;
            for (int q = 3; q < 16; ++q) pn[q] = __float2bfloat16_rn(0.f);
        }
        const float delta = __double2float_ru(sqrt(te) * (1.0 + 1e-12));
        atomicMax(&hstat[2 * h], __float_as_uint(delta));
        atomicMax(&hstat[2 * h + 1], __float_as_uint(__double2float_ru(tn)));
    }
}

static_assert(ALayout<128, true>::SMEM <= 232448 && ALayout<128, false>::SMEM <= 232448,
              "assignment kernel exceeds the shared memory of a block");

template <int D, bool FOLD>
cudaError_t launch_mma(const FastAssignArgs &a, const AsgParams &p, int grid, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(k_assign_mma<D, FOLD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)ALayout<D, FOLD>::SMEM);
    if (e != cudaSuccess) return e;
    k_assign_mma<D, FOLD><<<grid, A_THREADS, ALayout<D, FOLD>::SMEM, s>>>(*a.tm_x, *a.tm_c, FOLD ? *a.tm_cn : *a.tm_c, p);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_row_sqnorm(const bf16 *X, int64_t rows, int d, float *out, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    k_row_sqnorm<<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(X, rows, d, out);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

cudaError_t launch_assign_fast(const FastAssignArgs &a, cudaStream_t s) {
    cudaError_t e;
    const int BH = a.BH;
    if (BH <= 0 || a.L <= 0) return cudaSuccess;
    // 1. split the centres
    if ((e = cudaMemsetAsync(a.hstat, 0, sizeof(unsigned int) * 2 * BH, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(a.amb_count, 0, 2 * sizeof(int), s)) != cudaSuccess) return e;
    const bool fold = !a.two_term;
    k_centre_prep<<<dim3(a.Cpad, BH), 64, 0, s>>>(a.C, a.cstride, a.ncent, a.ncent_const, a.d, a.Cpad,
                                                  a.two_term ? 1 : 0, fold ? 1 : 0, a.Chi, a.cnp, a.cn, a.hstat);
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 2. tensor-core pass with the top-4 epilogue
    AsgParams p;
    p.inv = a.inv;
    p.rowsq = a.rowsq;
    p.cn = a.cn;
    p.hstat = a.hstat;
    p.nrows = a.nrows;
    p.nrows_const = a.nrows_const;
    p.ncent = a.ncent;
    p.ncent_const = a.ncent_const;
    p.L = a.L;
    p.BH = BH;
    p.Cpad = a.Cpad;
    p.CH = a.CH;
    p.units_per_head = (int)((a.L + AU - 1) / AU);
    p.two_term = a.two_term ? 1 : 0;
    // products * 2^-23; with the folded |c'|^2 the accumulated terms also sum |c'|^2,
    // so (d + 16) products at twice the rate
    p.e_tc = a.two_term ? (float)(2 * a.d) * 1.1920928955078125e-07f : (float)(a.d + 16) * 2.384185791015625e-07f;
    p.labels = a.labels;
    p.cand = a.cand;
    p.amb_list = a.amb_list;
    p.amb_count = a.amb_count;
    p.amb_cap = (int64_t)BH * a.L;
    p.stats = a.stats;
    p.err = a.err;
    p.c_stage = (uint32_t)(a.two_term ? 2 * (a.d / 64) * a.CH * 128 : (a.d / 64) * a.CH * 128 + a.CH * 32);
    p.nc = A_NC;
    // the centre stages must fit their region of shared memory
    const uint64_t region = a.two_term ? (uint64_t)A_NC * 2 * (a.d / 64) * QCH * 128
                                       : (uint64_t)A_NC * ((a.d / 64) * ACH * 128 + ACH * 32);
    if (a.CH < 32 || a.CH > ACH || (a.CH & 31) || (a.two_term && a.CH > QCH) || (a.Cpad & 31) ||
        (uint64_t)p.nc * p.c_stage > region)
        return cudaErrorInvalidValue;
    const int nunits = BH * p.units_per_head;
    const int grid = nunits < a.num_sms ? nunits : a.num_sms;
    if (fold) e = a.d == 128 ? launch_mma<128, true>(a, p, grid, s) : launch_mma<64, true>(a, p, grid, s);
    else e = a.d == 128 ? launch_mma<128, false>(a, p, grid, s) : launch_mma<64, false>(a, p, grid, s);
    if (e != cudaSuccess) return e;
    // 3. exact rescoring of the uncertain rows
    if (a.inv) {
        k_assign_resolve<true><<<4 * a.num_sms, 256, 0, s>>>(a.X, a.inv, a.L, a.d, a.C, a.cstride, a.cand,
                                                             a.amb_list, a.amb_count, a.labels, a.stats);
        k_assign_resolve_all<true><<<4 * a.num_sms, 256, 0, s>>>(a.X, a.inv, a.L, a.d, a.C, a.cstride, a.ncent,
                                                                 a.ncent_const, a.amb_list, p.amb_cap, a.amb_count,
                                                                 a.labels);
    } else {
        k_assign_resolve<false><<<4 * a.num_sms, 256, 0, s>>>(a.X, a.inv, a.L, a.d, a.C, a.cstride, a.cand,
                                                              a.amb_list, a.amb_count, a.labels, a.stats);
        k_assign_resolve_all<false><<<4 * a.num_sms, 256, 0, s>>>(a.X, a.inv, a.L, a.d, a.C, a.cstride, a.ncent,
                                                                  a.ncent_const, a.amb_list, p.amb_cap,
                                                                  a.amb_count, a.labels);
    }
    AC_NOTE_LAUNCH();
    AC_NOTE_LAUNCH();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 4. exact distance to the chosen centre
    if (a.dmin) {
        const int maxn = a.nrows ? (int)a.L : a.nrows_const;
        const dim3 grid2((maxn + 127) / 128, BH);
        if (a.inv)
            k_exact_dmin<true><<<grid2, 128, 0, s>>>(a.X, a.inv, a.L, a.d, a.C, a.cstride, a.nrows, a.nrows_const,
                                                     a.ncent, a.ncent_const, a.labels, a.dmin);
        else
            k_exact_dmin<false><<<grid2, 128, 0, s>>>(a.X, a.inv, a.L, a.d, a.C, a.cstride, a.nrows,
                                                      a.nrows_const, a.ncent, a.ncent_const, a.labels, a.dmin);
        AC_NOTE_LAUNCH();
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace ac
