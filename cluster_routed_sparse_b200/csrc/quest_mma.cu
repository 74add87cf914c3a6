// quest_mma.cu -- TensorQuest (AdaCluster, arXiv 2604.18348, Sec. 3.2.3,
// Eq. (1) and Algorithm 2) on tcgen05 tensor cores, fused with the per-row
// top-k of Algorithm 3 line 9.
//
// Eq. (1) at cluster level: S[qc, kc] = sum_d max(c_d Kmax_d, c_d Kmin_d), c the
// fp32 centre of query cluster qc and Kmax / Kmin the per-dimension bounds of
// key cluster kc (exact bf16 member values).  As Kmax >= Kmin, the maximum is
// c_d Kmax_d when c_d >= 0 and c_d Kmin_d otherwise, so S = c+ . Kmax + c- . Kmin
// with c+ = max(c, 0), c- = min(c, 0): one GEMM of K = 2d.  Each of c+ and c-
// is split into bf16 c_hi + c_lo, so one CTA forms
//   S' = [c+_hi | c+_lo | c-_hi | c-_lo] . [Kmax | Kmax | Kmin | Kmin]^T
// for up to 128 query clusters (MMA M) against 64 key clusters per chunk (N).
// |S' - S| and the fp32 rounding of the definition's own evaluation are
// bounded by E = eps(d) |c|_1 max_d max(|Kmax_d|, |Kmin_d|) (see quest_eps).
// The selection then stays exact: theta = the k-th largest lower bound S' - E
// over the non-empty clusters; every cluster whose upper bound S' + E is below
// theta has k clusters strictly above it, so the top-k lies in the candidate
// set R = {S' + E >= theta}.  When |R| = k, R is the selection; otherwise the
// scores of R are recomputed with the definition's arithmetic (fp32, products
// rounded, summed in dimension order) and the top-k of R is taken with ties to
// the lower cluster id -- the oracle's selection, bit for bit.
//
// Phase 1 (tensor cores), 512 threads:
//   warps 0-3  build the A operand (one query cluster per thread), then per
//              chunk the column bounds max |K| from the staged tile and the
//              scores from tensor memory (thread = TMEM lane = query cluster)
//   warp 4     TMA producer of the Kmax / Kmin chunks (two stages)
//   warp 5     tensor-memory owner and single-thread MMA issuer
// Phase 2 (selection), one warp per query cluster: the row's scores are staged
// in shared memory, radix-selected (8-bit digits), rescored where needed, and
// written out with the key ranges the attention kernel walks.  A CTA selects
// for 16 query clusters, so a head's selection spreads over several SMs; each
// of them recomputes the head's (small) score GEMM and writes its own rows.
#include <algorithm>

#include "ac_device.cuh"
#include "ac_internal.h"

namespace ac {
namespace {

constexpr int QM = 128;          // query clusters per MMA tile (M)
constexpr int QR = 16;           // query clusters a CTA selects for (one per warp); the CTAs
                                 // of one MMA tile each recompute its small GEMM
constexpr int QN = 64;           // key clusters per chunk (MMA N)
constexpr int Q_STAGES = 2;
constexpr int Q_THREADS = 512;
constexpr int Q_WARPS = Q_THREADS / 32;
constexpr int Q_EPI = 128;       // epilogue threads of phase 1

template <int D>
struct QLayout {
    static constexpr int HALVES = D / 64;
    static constexpr uint32_t A_BLK = QM * D * 2;     // one term: [8-row group][16-byte column][8 rows][16 B]
    static constexpr uint32_t OFF_A = 0;              // c+_hi, c+_lo, c-_hi, c-_lo
    static constexpr uint32_t KT = HALVES * QN * 128;  // one Kmax (or Kmin) chunk: [half][QN rows][128 B], swizzled
    static constexpr uint32_t OFF_B = OFF_A + 4 * A_BLK;
    static constexpr uint32_t STAGE = 2 * KT;
    static constexpr uint32_t OFF_BAR = OFF_B + Q_STAGES * STAGE;
    static constexpr uint32_t P1_BYTES = OFF_BAR + 128;
};

enum { QB_F = 0, QB_E = 2, QB_AF = 4, QB_AE = 6, QB_AR = 8, QB_DONE = 9, QB_N = 10 };

// Relative error coefficient of S' (and of the definition's fp32 evaluation)
// against the exact sum, in units of |c|_1 max|K|:
//   2^-16                the bf16 split: |c - c_hi - c_lo| <= 2^-16 |c|;
//   4d 2^-23 (1 + 2^-7)  the tensor core's fp32 accumulation of the 4d exact
//                        products, allowed two units in the last place per
//                        addition, of terms summing to at most (1 + 2^-7) sum|c||K|;
//   (d + 1) 2^-24        the definition itself: d rounded products, d - 1 sums;
// widened by 2^-10 for the fp32 evaluation of the bound.
__host__ __device__ constexpr float quest_eps(int d) {
    return (1.52587890625e-05f + 4.0f * d * 1.1920928955078125e-07f * 1.0078125f +
            (d + 1) * 5.9604644775390625e-08f) * 1.0009765625f;
}

struct QuestParams {
    const float *cent_q;      // [BH, Cq, d]
    const bf16 *kmax, *kmin;  // [BH, Ccap, d]
    const int *counts_k;      // [BH, Ccap]
    const int *n_k;           // [BH]
    const uint8_t *dense;     // [BH]
    const int *pgoff;         // [BH, Ccap]
    float *score;             // [BH, Cq, Ccap]
    float *kabs;              // [BH, Ccap] column bounds max_d max(|Kmax_d|, |Kmin_d|)
    int *sel, *ksel, *nrange, *nboxes, *rbox;
    int2 *ranges;
    uint32_t *err;
    float *cbias;       // centroid compensation (null: off): [BH, Cq, Ccap] addends, crange [BH*Cq]
    int *crange;
    int cgroup;
    float scale;
    float bound_scale;  // >= 1: widens E (more candidates rescored; the selection is unchanged)
    int Cq, Ccap, BH, topk, warps2;
};

__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);  // both zeros: one key
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// One 8-bit digit pass of a most-significant-first radix select by one warp:
// among the entries whose key matches `prefix` on the bits above `shift`,
// find the digit of the need-th largest key.  hist: 256 words of the warp.
__device__ __forceinline__ void warp_digit(uint32_t *hist, int shift, uint32_t &prefix, uint32_t &above,
                                           uint32_t need_total) {
    const int lane = threadIdx.x & 31;
    // lane l owns the digits 255 - 8l .. 248 - 8l (descending)
    uint32_t h[8], s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        h[i] = hist[255 - 8 * lane - i];
        s += h[i];
    }
    uint32_t incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += t;
    }
    const uint32_t need = need_total - above;
    const uint32_t hit = __ballot_sync(0xFFFFFFFFu, incl >= need);
    const int L = __ffs(hit) - 1;  // need >= 1 and the histogram holds enough entries
    uint32_t cum = incl - s, dg = 0;
    if (lane == L) {
        dg = 255 - 8 * lane - 7;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (cum + h[i] >= need) {
                dg = 255 - 8 * lane - i;
                break;
            }
            cum += h[i];
        }
    }
    dg = __shfl_sync(0xFFFFFFFFu, dg, L);
    cum = __shfl_sync(0xFFFFFFFFu, cum, L);
    above += cum;
    prefix = (prefix << 8) | dg;
    (void)shift;
}

template <int D>
__global__ void __launch_bounds__(Q_THREADS, 1)
    k_quest_select_mma(const __grid_constant__ CUtensorMap tm_kmax, const __grid_constant__ CUtensorMap tm_kmin,
                       const QuestParams p) {
    using LY = QLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // this CTA's query clusters r_lo .. r_hi - 1, inside the MMA tile of rows m0 ..
    const int h = blockIdx.x, r_lo = blockIdx.y * QR, r_hi = min(p.Cq, r_lo + QR);
    const int m0 = (r_lo / QM) * QM;
    const int rows = min(QM, p.Cq - m0);
    const int nk = p.n_k[h];
    const int nch = (nk + QN - 1) / QN;
    const uint32_t bar0 = sbase + LY::OFF_BAR;
#define QBAR(i) (bar0 + 8u * (uint32_t)(i))
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + LY::OFF_BAR + 8 * QB_N);
    const float *cq = p.cent_q + ((int64_t)h * p.Cq + m0) * D;
    const int *cnt = p.counts_k + (int64_t)h * p.Ccap;

    if (tid == 0) {
        for (int i = 0; i < Q_STAGES; ++i) {
            mbar_init(QBAR(QB_F + i), 1);
            mbar_init(QBAR(QB_E + i), 1 + Q_EPI);  // the MMAs' commit and the column-bound readers
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(QBAR(QB_AF + i), 1);
            mbar_init(QBAR(QB_AE + i), Q_EPI);
        }
        mbar_init(QBAR(QB_AR), Q_EPI);
        mbar_init(QBAR(QB_DONE), 1);
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_slot), 2 * QN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    // ============================================================ phase 1
    if (nch > 0) {
        if (warp == 4) {
            if (lane == 0) {
                for (int ch = 0; ch < nch; ++ch) {
                    const int s = ch % Q_STAGES;
                    if (ch >= Q_STAGES &&
                        !mbar_wait_or_abort(QBAR(QB_E + s), ((ch / Q_STAGES) - 1) & 1, p.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = sbase + LY::OFF_B + s * LY::STAGE;
                    mbar_arrive_expect_tx(QBAR(QB_F + s), LY::STAGE);
                    const int row = h * p.Ccap + ch * QN;
                    for (int hf = 0; hf < LY::HALVES; ++hf) {
                        tma_load_2d(dst + hf * QN * 128, &tm_kmax, hf * 64, row, QBAR(QB_F + s));
                        tma_load_2d(dst + LY::KT + hf * QN * 128, &tm_kmin, hf * 64, row, QBAR(QB_F + s));
                    }
                }
                // nothing may still be landing when the block moves on
                for (int ch = max(0, nch - Q_STAGES); ch < nch; ++ch)
                    if (!mbar_wait(QBAR(QB_F + ch % Q_STAGES), (ch / Q_STAGES) & 1)) ok = false;
                if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
            }
            __syncwarp();
        } else if (warp == 5) {
            if (lane == 0) {
                constexpr uint32_t IDESC = idesc_bf16_f32(QM, QN, false);
                if (!mbar_wait_or_abort(QBAR(QB_AR), 0, p.err)) ok = false;
                for (int ch = 0; ch < nch && ok; ++ch) {
                    const int s = ch % Q_STAGES, a = ch & 1;
                    if (!mbar_wait_or_abort(QBAR(QB_F + s), (ch / Q_STAGES) & 1, p.err) ||
                        (ch >= 2 && !mbar_wait_or_abort(QBAR(QB_AE + a), ((ch >> 1) - 1) & 1, p.err))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t bs = sbase + LY::OFF_B + s * LY::STAGE;
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) {
                        const uint32_t ab = sbase + LY::OFF_A + blk * LY::A_BLK;
                        const uint32_t kb = bs + (blk < 2 ? 0u : LY::KT);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            tc_mma_bf16(tmem + a * QN, sdesc_noswz(ab + kk * 256, 128, (D / 8) * 128),
                                        sdesc_sw128(kb + (kk >> 2) * (QN * 128) + (kk & 3) * 32, 16, 1024), IDESC,
                                        (blk | kk) ? 1u : 0u);
                        }
                    }
                    tc_commit(QBAR(QB_AF + a));
                    tc_commit(QBAR(QB_E + s));
                }
                tc_commit(QBAR(QB_DONE));
                if (!mbar_wait(QBAR(QB_DONE), 0)) ok = false;
                if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
            }
            __syncwarp();
        } else if (warp < 4) {
            const int r = tid;  // query cluster m0 + r, TMEM lane r
            // ---- A operand: c+ and c- split into bf16 hi + lo, core-matrix layout
            {
                uint8_t *A = sm + LY::OFF_A;
                const int g = r >> 3, rr = r & 7;
                for (int j = 0; j < D / 8; ++j) {
                    float v[8];
                    if (r < rows) {
                        const float4 *src = reinterpret_cast<const float4 *>(cq + (int64_t)r * D + 8 * j);
                        const float4 x0 = src[0], x1 = src[1];
                        v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
                        v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
                    } else {
#pragma unroll
                        for (int i = 0; i < 8; ++i) v[i] = 0.f;
                    }
                    uint32_t w[4][4];
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        float t[4][2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float pp = v[i + e] > 0.f ? v[i + e] : 0.f;
                            const float nn = v[i + e] < 0.f ? v[i + e] : 0.f;
                            const float ph = __bfloat162float(__float2bfloat16_rn(pp));
                            const float nh = __bfloat162float(__float2bfloat16_rn(nn));
                            t[0][e] = ph;
                            t[1][e] = pp - ph;  // exact in fp32
                            t[2][e] = nh;
                            t[3][e] = nn - nh;
                        }
#pragma unroll
                        for (int b = 0; b < 4; ++b) w[b][i >> 1] = pack_bf16x2(t[b][0], t[b][1]);
                    }
                    const uint32_t off = (uint32_t)(g * (D / 8) + j) * 128u + rr * 16u;
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        *reinterpret_cast<uint4 *>(A + b * LY::A_BLK + off) = make_uint4(w[b][0], w[b][1], w[b][2], w[b][3]);
                }
                fence_proxy_async_smem();
                mbar_arrive(QBAR(QB_AR));
            }
            const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
            float *srow = p.score + ((int64_t)h * p.Cq + m0 + r) * p.Ccap;
            for (int ch = 0; ch < nch; ++ch) {
                const int s = ch % Q_STAGES, a = ch & 1;
                // ---- column bounds of this chunk: the two threads of a lane pair
                // read the two column halves of one key cluster's Kmax and Kmin rows
                // (the 128-byte swizzle only permutes 16-byte pieces within a row)
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_or_abort(QBAR(QB_F + s), (ch / Q_STAGES) & 1, p.err))) {
                    ok = false;
                    break;
                }
                const int col = r >> 1, hf = r & 1;
                uint32_t mx = 0u;
                if (hf < LY::HALVES) {
                    const uint8_t *base = sm + LY::OFF_B + s * LY::STAGE + hf * QN * 128 + col * 128;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(base + t * LY::KT + q * 16);
                            const uint32_t ws[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                mx = max(mx, max(ws[e] & 0x7FFFu, (ws[e] >> 16) & 0x7FFFu));
                        }
                    }
                }
                mbar_arrive(QBAR(QB_E + s));
                mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
                if (hf == 0 && ch * QN + col < nk) p.kabs[(int64_t)h * p.Ccap + ch * QN + col] = __uint_as_float(mx << 16);
                // ---- scores of this chunk from tensor memory
                if (!__all_sync(0xFFFFFFFFu, mbar_wait_or_abort(QBAR(QB_AF + a), (ch >> 1) & 1, p.err))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t v[2][32];
                tmem_ld32(tmem + lane_off + a * QN, v[0]);
                tmem_ld32(tmem + lane_off + a * QN + 32, v[1]);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(QBAR(QB_AE + a));
                if (m0 + r >= r_lo && m0 + r < r_hi) {
                    const int c0 = ch * QN;
#pragma unroll
                    for (int q = 0; q < 2; ++q)
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int c = c0 + 32 * q + i;
                            if (c < nk) srow[c] = cnt[c] != 0 ? __uint_as_float(v[q][i]) : -INFINITY;
                        }
                }
            }
            if (!ok) set_err(p.err, DEV_ERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    ok = __syncthreads_and(ok);
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * QN);
    }
    if (!ok) return;  // a bounded wait expired: the selection keeps its previous contents

    // ============================================================ phase 2
    // shared memory, reused: query centres [rows][D] | column bounds [Ccap] |
    // non-empty bits [W] | per warp: scores [Ccap], histogram [256], R bits [W], selected bits [W]
    const int W = (p.Ccap + 31) / 32;
    float *cq_s = reinterpret_cast<float *>(sm);
    float *kb_s = cq_s + QM * D;
    uint32_t *ne_s = reinterpret_cast<uint32_t *>(kb_s + p.Ccap);
    uint8_t *wbase = reinterpret_cast<uint8_t *>(ne_s + W);
    const size_t per_warp = (size_t)p.Ccap * 4 + 1024 + 8 * (size_t)W;
    for (int i = tid; i < rows * D; i += Q_THREADS) cq_s[i] = cq[i];
    for (int c = tid; c < nk; c += Q_THREADS) kb_s[c] = p.kabs[(int64_t)h * p.Ccap + c];
    for (int wi = tid; wi < W; wi += Q_THREADS) {
        uint32_t b = 0u;
        for (int i = 0; i < 32; ++i) {
            const int c = wi * 32 + i;
            b |= (c < nk && cnt[c] != 0) ? (1u << i) : 0u;
        }
        ne_s[wi] = b;
    }
    __syncthreads();
    if (warp >= p.warps2) return;
    float *Sw = reinterpret_cast<float *>(wbase + warp * per_warp);
    uint32_t *hist = reinterpret_cast<uint32_t *>(Sw + p.Ccap);
    uint32_t *rbits = hist + 256;
    uint32_t *sbits = rbits + W;
    const int nw = (nk + 31) / 32;
    int ne = 0;
    for (int wi = lane; wi < nw; wi += 32) ne += __popc(ne_s[wi]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ne += __shfl_xor_sync(0xFFFFFFFFu, ne, o);
    int64_t kk64 = p.topk > 0 ? p.topk : ((int64_t)(-p.topk) * nk + 999) / 1000;
    if (kk64 > ne) kk64 = ne;
    if (kk64 < 1) kk64 = 1;
    const int k = (int)kk64;
    if (blockIdx.y == 0 && warp == 0 && lane == 0) p.ksel[h] = k;
    const bool dense = p.dense[h] != 0;
    const int *pg = p.pgoff + (int64_t)h * p.Ccap;
    const float eps = quest_eps(D);

    for (int r = r_lo - m0 + warp; r < r_hi - m0; r += p.warps2) {
        const int64_t hq = (int64_t)h * p.Cq + m0 + r;
        float *srow = p.score + hq * p.Ccap;
        for (int c = lane; c < nk; c += 32) Sw[c] = srow[c];
        // E for this row: eps |c|_1 (|c|_1 in fp32, widened for its own rounding)
        float l1 = 0.f;
        for (int i = lane; i < D; i += 32) l1 += fabsf(cq_s[r * D + i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, o);
        const float erow = eps * l1 * (1.f + D * 1.2e-7f) * p.bound_scale;
        __syncwarp();
        int nsel = 0;  // entries of sbits set
        // ---- theta: the k-th largest lower bound among the non-empty clusters
        uint32_t prefix = 0u, above = 0u;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = lane; i < 256; i += 32) hist[i] = 0u;
            __syncwarp();
            for (int c = lane; c < nk; c += 32) {
                if (!((ne_s[c >> 5] >> (c & 31)) & 1u)) continue;
                const float sv = Sw[c];
                const float e = erow * kb_s[c] + fabsf(sv) * 4.76837158203125e-07f;
                const uint32_t key = order_key(sv - e);
                if (shift == 24 || (key >> (shift + 8)) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
            }
            __syncwarp();
            warp_digit(hist, shift, prefix, above, (uint32_t)k);
            __syncwarp();
        }
        const float theta = key_float(prefix);
        // ---- candidates R: upper bound >= theta
        int nR = 0;
        for (int c0 = 0; c0 < nw * 32; c0 += 32) {
            const int c = c0 + lane;
            bool in = false;
            if (c < nk && ((ne_s[c >> 5] >> (c & 31)) & 1u)) {
                const float sv = Sw[c];
                const float e = erow * kb_s[c] + fabsf(sv) * 4.76837158203125e-07f;
                in = sv + e >= theta;
            }
            const uint32_t b = __ballot_sync(0xFFFFFFFFu, in);
            if (lane == 0) rbits[c0 >> 5] = b;
            nR += __popc(b);
        }
        __syncwarp();
        if (nR == k) {
            for (int wi = lane; wi < nw; wi += 32) sbits[wi] = rbits[wi];
            nsel = k;
        } else {
            // ---- rescore R with the definition's arithmetic
            const bf16 *kx = p.kmax + (int64_t)h * p.Ccap * D, *kn = p.kmin + (int64_t)h * p.Ccap * D;
            for (int c = lane; c < nw * 32; c += 32) {
                if (!((rbits[c >> 5] >> (c & 31)) & 1u)) continue;
                float acc = 0.f;
                const bf16 *xr = kx + (int64_t)c * D, *nr = kn + (int64_t)c * D;
                for (int d = 0; d < D; ++d) {
                    const float qd = cq_s[r * D + d];
                    const float u = __fmul_rn(qd, bf2f(xr[d]));
                    const float w = __fmul_rn(qd, bf2f(nr[d]));
                    acc = __fadd_rn(acc, u > w ? u : w);
                }
                Sw[c] = acc;
                srow[c] = acc;
            }
            __syncwarp();
            prefix = 0u;
            above = 0u;
            for (int shift = 24; shift >= 0; shift -= 8) {
                for (int i = lane; i < 256; i += 32) hist[i] = 0u;
                __syncwarp();
                for (int c = lane; c < nk; c += 32) {
                    if (!((rbits[c >> 5] >> (c & 31)) & 1u)) continue;
                    const uint32_t key = order_key(Sw[c]);
                    if (shift == 24 || (key >> (shift + 8)) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
                }
                __syncwarp();
                warp_digit(hist, shift, prefix, above, (uint32_t)k);
                __syncwarp();
            }
            // keep every key above K*, and of those equal to K* the lowest ids
            const int need_eq = k - (int)above;
            int eq_before = 0;
            for (int c0 = 0; c0 < nw * 32; c0 += 32) {
                const int c = c0 + lane;
                const bool inr = (rbits[c0 >> 5] >> lane) & 1u;
                const uint32_t key = inr ? order_key(Sw[c]) : 0u;
                const bool gt = inr && key > prefix, eq = inr && key == prefix;
                const uint32_t be = __ballot_sync(0xFFFFFFFFu, eq);
                const int pos = eq_before + __popc(be & ((1u << lane) - 1u));
                const bool take = gt || (eq && pos < need_eq);
                const uint32_t bt = __ballot_sync(0xFFFFFFFFu, take);
                if (lane == 0) sbits[c0 >> 5] = bt;
                eq_before += __popc(be);
            }
            nsel = k;
        }
        __syncwarp();
        // ---- the selection in ascending id order, and the key ranges to walk
        int *selrow = p.sel + hq * p.Ccap;
        int2 *rg = p.ranges + hq * p.Ccap;
        int *rb = p.rbox + hq * (p.Ccap + 1);
        int spos = 0, rpos = 0, gpos = 0;
        for (int c0 = 0; c0 < nw * 32; c0 += 32) {
            const int c = c0 + lane;
            const bool s = (sbits[c0 >> 5] >> lane) & 1u;
            const uint32_t bs = __ballot_sync(0xFFFFFFFFu, s);
            if (s) selrow[spos + __popc(bs & ((1u << lane) - 1u))] = c;
            spos += __popc(bs);
            const bool nonempty = (ne_s[c0 >> 5] >> lane) & 1u;
            const bool walk = dense ? nonempty : s;
            const uint32_t bw = __ballot_sync(0xFFFFFFFFu, walk);
            const int cc = walk ? cnt[c] : 0;
            int g = (cc + 7) / 8, incl = g;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += t;
            }
            if (walk) {
                const int ri = rpos + __popc(bw & ((1u << lane) - 1u));
                rg[ri] = make_int2(pg[c], cc);
                rb[ri] = gpos + incl - g;
            }
            rpos += __popc(bw);
            gpos += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        // centroid compensation: the unselected non-empty clusters as pseudo-keys
        // (one more range, over the centroid block), with their addends ln|c| / scale
        if (p.cbias) {
            float *cb = p.cbias + hq * p.Ccap;
            for (int c = lane; c < nk; c += 32) {
                const bool sl = (sbits[c >> 5] >> (c & 31)) & 1u;
                const bool nz = (ne_s[c >> 5] >> (c & 31)) & 1u;
                cb[c] = (sl || !nz) ? -INFINITY : logf((float)cnt[c]) / p.scale;
            }
        }
        if (lane == 0) {
            if (p.cbias && !dense && ne > k) {
                rg[rpos] = make_int2(p.cgroup, nk);
                rb[rpos] = gpos;
                p.crange[hq] = rpos;
                ++rpos;
                gpos += (nk + 7) / 8;
            } else if (p.crange) {
                p.crange[hq] = -1;
            }
            p.nrange[hq] = rpos;
            p.nboxes[hq] = gpos;
            rb[rpos] = gpos;
        }
        (void)nsel;
        __syncwarp();
    }
#undef QBAR
}

template <int D>
size_t quest_p2_bytes(int Ccap, int warps) {
    const int W = (Ccap + 31) / 32;
    return (size_t)QM * D * 4 + (size_t)Ccap * 4 + 4 * (size_t)W + (size_t)warps * ((size_t)Ccap * 4 + 1024 + 8 * (size_t)W);
}

template <int D>
cudaError_t launch_quest_d(const SelectArgs &a, cudaStream_t s) {
    using LY = QLayout<D>;
    constexpr size_t kMaxSmem = 227 * 1024 - 1024;  // less the alignment slack
    int warps = Q_WARPS;
    while (warps > 1 && quest_p2_bytes<D>(a.Ccap, warps) > kMaxSmem) --warps;
    const size_t bytes = std::max<size_t>(LY::P1_BYTES, quest_p2_bytes<D>(a.Ccap, warps));
    if (bytes > kMaxSmem) return cudaErrorInvalidValue;
    QuestParams p;
    p.cent_q = a.cent_q;
    p.kmax = a.kmax;
    p.kmin = a.kmin;
    p.counts_k = a.counts_k;
    p.n_k = a.n_k;
    p.dense = a.dense;
    p.pgoff = a.pgoff;
    p.score = a.score;
    p.kabs = a.kabs;
    p.sel = a.sel;
    p.ksel = a.ksel;
    p.nrange = a.nrange;
    p.nboxes = a.nboxes;
    p.rbox = a.rbox;
    p.ranges = a.ranges;
    p.err = a.err;
    p.bound_scale = a.bound_scale >= 1.f ? a.bound_scale : 1.f;
    p.cbias = a.cbias;
    p.crange = a.crange;
    p.cgroup = a.cgroup;
    p.scale = a.scale;
    p.Cq = a.Cq;
    p.Ccap = a.Ccap;
    p.BH = a.BH;
    p.topk = a.topk;
    p.warps2 = warps;
    const int smem = (int)(bytes + 1024);
    cudaError_t e = cudaFuncSetAttribute(k_quest_select_mma<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k_quest_select_mma<D><<<dim3(a.BH, (a.Cq + QR - 1) / QR), Q_THREADS, smem, s>>>(*a.tm_kmax, *a.tm_kmin, p);
    AC_NOTE_LAUNCH();
    return cudaGetLastError();
}

}  // namespace

bool quest_mma_supported(const SelectArgs &a) {
    if (a.score_mode != 0 || !a.tm_kmax || !a.tm_kmin || !a.kabs) return false;
    if (a.d != 64 && a.d != 128) return false;
    return true;
}

cudaError_t launch_quest_select_mma(const SelectArgs &a, cudaStream_t s) {
    return a.d == 128 ? launch_quest_d<128>(a, s) : launch_quest_d<64>(a, s);
}

}  // namespace ac
