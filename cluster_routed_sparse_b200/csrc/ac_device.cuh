// ac_device.cuh -- device helpers for sm_100a: bf16 conversion, the seeded
// counter-based generator, bounded mbarrier waits, TMA and tcgen05 wrappers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ac {

// ------------------------------------------------------------------ errors
// Error word written by kernels (never trap on the device).
enum : uint32_t {
    DEV_ERR_TIMEOUT = 1u,     // a bounded wait expired
    DEV_ERR_BOUNDS = 2u,      // an index failed its bounds check
    DEV_ERR_NONFINITE = 4u,   // NaN / Inf met in an input
};

__device__ __forceinline__ void set_err(uint32_t *err, uint32_t bit) {
    if (err) atomicOr(err, bit);
}

// ------------------------------------------------------------------ numbers
__device__ __forceinline__ float bf2f(__nv_bfloat16 v) { return __bfloat162float(v); }

// SplitMix64 output function (Steele, Lea, Flood, OOPSLA 2014).
__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// The (i+1)-th SplitMix64 output of a generator keyed by (seed, unit, tag).
__device__ __forceinline__ uint64_t seeded_rand(uint64_t seed, int64_t unit, int32_t tag, int64_t i) {
    uint64_t key = mix64(seed ^ mix64((((uint64_t)unit) << 32) ^ (uint64_t)(uint32_t)tag));
    return mix64(key + (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ull);
}

// Member chosen for initial centre j of m among n (j-th of m equal strata).
__device__ __forceinline__ int64_t stratum_pick(uint64_t seed, int64_t unit, int32_t tag, int64_t n,
                                                int32_t m, int32_t j) {
    int64_t lo = ((int64_t)j * n) / m;
    int64_t hi = ((int64_t)(j + 1) * n) / m;
    return lo + (int64_t)(seeded_rand(seed, unit, tag, j) % (uint64_t)(hi - lo));
}

// ------------------------------------------------------------------ time
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ smem / mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for a bounded time.
// Three independent bounds: SM cycles (clock64), nanoseconds (%globaltimer)
// and a poll count, so the wait ends even if one clock does not advance.
// Returns false when a bound is hit (the caller records the error and leaves
// its loop; no thread ever spins without bound).
constexpr uint64_t kWaitLimitNs = 2000000000ull;     // 2 s
constexpr long long kWaitLimitCycles = 4000000000ll;  // ~2 s at 2 GHz
constexpr uint32_t kWaitLimitPolls = 1u << 24;

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const long long c0 = clock64();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u &&
            (globaltimer_ns() - t0 > kWaitLimitNs || clock64() - c0 > kWaitLimitCycles || it > kWaitLimitPolls))
            return false;
    }
}

// As mbar_wait with a caller-chosen time limit (limit_ns, at most kWaitLimitNs);
// the cycle bound is 4 cycles per nanosecond of the limit, the poll bound the
// same as mbar_wait's.
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (limit_ns > kWaitLimitNs) limit_ns = kWaitLimitNs;
    const long long cycle_limit = (long long)limit_ns * 4;
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const long long c0 = clock64();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u &&
            (globaltimer_ns() - t0 > limit_ns || clock64() - c0 > cycle_limit || it > kWaitLimitPolls))
            return false;
    }
}

// As mbar_wait, but also gives up as soon as another CTA has recorded an error
// in *abort (so one stuck CTA does not make every CTA sit out its own limit).
__device__ __forceinline__ bool mbar_wait_or_abort(uint32_t bar, uint32_t parity, const uint32_t *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const long long c0 = clock64();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u) {
            if (abort && *reinterpret_cast<const volatile uint32_t *>(abort) != 0u) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs || clock64() - c0 > kWaitLimitCycles || it > kWaitLimitPolls)
                return false;
        }
    }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMA
// 2-D tiled bulk tensor load into shared memory, completion counted on `bar`.
// x is the innermost (column) coordinate, y the row.  No cluster multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int32_t x, int32_t y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// 4-D tiled bulk tensor load (coordinates x innermost).  No cluster multicast.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void *tmap, int32_t x, int32_t y, int32_t z,
                                            int32_t w, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar)
        : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_slot),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A (M x K bf16) read from tensor memory, one
// row per lane, two consecutive K elements per 32-bit column.
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Eight tcgen05.mma (SS) into one accumulator in one asm block, for issuing
// threads that share their sub-partition with busy warps.  Product 0 takes the
// descriptors as given, product k = 1..7 adds Ak to the low word of A's and Bk
// to the low word of B's (offsets in 16-byte units; the caller keeps every
// operand inside shared memory, so the 14-bit address field does not carry).
// Product 0 accumulates when acc != 0, the others always.
template <uint32_t A1, uint32_t A2, uint32_t A3, uint32_t A4, uint32_t A5, uint32_t A6, uint32_t A7,
          uint32_t B1, uint32_t B2, uint32_t B3, uint32_t B4, uint32_t B5, uint32_t B6, uint32_t B7>
__device__ __forceinline__ void mma8_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t.reg .b32 alo, ahi, blo, bhi, x, y;\n\t.reg .b64 da, db;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, %4, %4;\n\t"
        "mov.b64 {alo, ahi}, %1;\n\tmov.b64 {blo, bhi}, %2;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "add.u32 x, alo, %5;\n\tadd.u32 y, blo, %12;\n\tmov.b64 da, {x, ahi};\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, t;\n\t"
        "add.u32 x, alo, %6;\n\tadd.u32 y, blo, %13;\n\tmov.b64 da, {x, ahi};\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, t;\n\t"
        "add.u32 x, alo, %7;\n\tadd.u32 y, blo, %14;\n\tmov.b64 da, {x, ahi};\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, t;\n\t"
        "add.u32 x, alo, %8;\n\tadd.u32 y, blo, %15;\n\tmov.b64 da, {x, ahi};\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, t;\n\t"
        "add.u32 x, alo, %9;\n\tadd.u32 y, blo, %16;\n\tmov.b64 da, {x, ahi};\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, t;\n\t"
        "add.u32 x, alo, %10;\n\tadd.u32 y, blo, %17;\n\tmov.b64 da, {x, ahi};\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, t;\n\t"
        "add.u32 x, alo, %11;\n\tadd.u32 y, blo, %18;\n\tmov.b64 da, {x, ahi};\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %3, t;\n\t}"
        ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "n"(A1), "n"(A2), "n"(A3), "n"(A4), "n"(A5),
        "n"(A6), "n"(A7), "n"(B1), "n"(B2), "n"(B3), "n"(B4), "n"(B5), "n"(B6), "n"(B7)
        : "memory");
}

// Eight tcgen05.mma (TS: A from tensor memory at a + 8 k columns) into one
// accumulator; B descriptor k is {b_lo + B_STEP * k, b_hi}.
template <uint32_t B_STEP>
__device__ __forceinline__ void mma8_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t.reg .b32 blo, bhi, y, ta;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, %4, %4;\n\t"
        "mov.b64 {blo, bhi}, %2;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "add.u32 y, blo, %5;\n\tadd.u32 ta, %1, 8;\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, t;\n\t"
        "add.u32 y, blo, %6;\n\tadd.u32 ta, %1, 16;\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, t;\n\t"
        "add.u32 y, blo, %7;\n\tadd.u32 ta, %1, 24;\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, t;\n\t"
        "add.u32 y, blo, %8;\n\tadd.u32 ta, %1, 32;\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, t;\n\t"
        "add.u32 y, blo, %9;\n\tadd.u32 ta, %1, 40;\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, t;\n\t"
        "add.u32 y, blo, %10;\n\tadd.u32 ta, %1, 48;\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, t;\n\t"
        "add.u32 y, blo, %11;\n\tadd.u32 ta, %1, 56;\n\tmov.b64 db, {y, bhi};\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %3, t;\n\t}"
        ::"r"(d), "r"(a), "l"(bdesc), "r"(idesc), "r"(acc), "n"(B_STEP), "n"(2 * B_STEP), "n"(3 * B_STEP),
        "n"(4 * B_STEP), "n"(5 * B_STEP), "n"(6 * B_STEP), "n"(7 * B_STEP)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// columns [col, col+32) of lane (warp quadrant base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// 32 lanes x 32 consecutive 32-bit columns from registers (thread i -> lane base + i).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05), 128-byte swizzle.
//   K-major operand: rows of 128 B, 8-row groups SBO = 1024 B apart.
//   MN-major operand: 64-element MN blocks LBO bytes apart, 8-row K groups
//   SBO bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100
    d |= (uint64_t)2 << 61;  // 128-byte swizzle
    return d;
}

// Shared-memory matrix descriptor (tcgen05), no swizzle, K-major: core
// matrices of 8 rows x 16 bytes stored contiguously (128 B); LBO = byte
// distance between core matrices along K, SBO = along M / N.
__device__ __forceinline__ uint64_t sdesc_noswz(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version for sm_100; layout type 0 = no swizzle
    return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 D, K-major A.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Per-warpgroup register budget (all 128 threads of the warpgroup execute it).
template <uint32_t N>
__device__ __forceinline__ void reg_alloc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void reg_dealloc() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pairs (sm_100): two IEEE operations per instruction, each
// rounded exactly like its scalar counterpart.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// min(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// max(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace ac
