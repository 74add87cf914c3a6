// noalloc.cu -- query clustering for callers that cannot allocate device memory.
//
// ac_cluster_q_noalloc does the work of ac_cluster_q (L2-normalise the
// queries, then Lloyd k-means on the unit vectors) without a context and
// without any device allocation.  Its scratch -- the inverse query norms, the
// cluster-order permutation and the per-cluster offsets and counts -- lives in
// one file-scope __device__ array of fixed size, which every GPU that loads
// libac holds until the process exits.  The caller supplies only the inputs and
// the outputs (labels and centres; the centres are updated in place) and,
// optionally, a device word that receives the kernels' error bits.
//
// Who needs this: code that runs where cudaMalloc is not allowed or not wise --
// inside a plugin's enqueue callback of an inference engine, in a server that
// must not grow its memory footprint while serving, or in a process whose
// device memory is entirely owned by another allocator.
#include <cuda.h>

#include <mutex>
#include <utility>
#include <vector>

#include "ac_device.cuh"
#include "ac_internal.h"

namespace {

constexpr int64_t kMaxRows = int64_t(1) << 20;  // B*H*L
constexpr int64_t kMaxCentreSlots = 1 << 16;    // B*H*(Cq+1)
constexpr int kMaxCq = 4096;                    // the stable sort keeps 8 histograms of Cq counts in shared memory

constexpr size_t kErrBytes = 256;  // one error word, padded to keep the arrays below aligned
constexpr size_t kInvBytes = sizeof(float) * kMaxRows;
constexpr size_t kPermBytes = sizeof(int) * kMaxRows;
constexpr size_t kOffsBytes = sizeof(int) * kMaxCentreSlots;
constexpr size_t kCountBytes = sizeof(int) * kMaxCentreSlots;
constexpr size_t kScratchBytes = kErrBytes + kInvBytes + kPermBytes + kOffsBytes + kCountBytes;  // 8.5 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch, looked up once per CUDA context (a
// context that was reset and created again gets a new id, hence a new lookup).
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

std::mutex g_mu;
std::vector<std::pair<unsigned long long, void *>> g_addr;  // (context id, address)
CtxGetCurrentFn g_get_current = nullptr;
CtxGetIdFn g_get_id = nullptr;

bool current_context_id(unsigned long long *id) {
    if (!g_get_current || !g_get_id) {
        void *p = nullptr, *q = nullptr;
        cudaDriverEntryPointQueryResult r1, r2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r1) != cudaSuccess ||
            r1 != cudaDriverEntryPointSuccess || !p ||
            cudaGetDriverEntryPoint("cuCtxGetId", &q, cudaEnableDefault, &r2) != cudaSuccess ||
            r2 != cudaDriverEntryPointSuccess || !q)
            return false;
        g_get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        g_get_id = reinterpret_cast<CtxGetIdFn>(q);
    }
    CUcontext ctx = nullptr;
    if (g_get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return g_get_id(ctx, id) == CUDA_SUCCESS;
}

cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_mu);
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    if (have_id)
        for (const auto &kv : g_addr)
            if (kv.first == id) {
                *out = kv.second;
                return cudaSuccess;
            }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // also makes the device's primary context current
    if (e != cudaSuccess) return e;
    if (have_id || current_context_id(&id)) g_addr.emplace_back(id, p);
    *out = p;
    return cudaSuccess;
}

}  // namespace

using namespace ac;

extern "C" ac_status ac_cluster_q_noalloc(const uint16_t *Q, int32_t BH, int32_t L, int32_t d, int32_t Cq,
                                          int32_t iters, uint64_t seed, const float *init_centroids,
                                          int32_t *labels_out, float *centroids_out, uint32_t *err_out,
                                          void *stream) {
    if (!Q || !labels_out || !centroids_out || BH < 1 || L < 1 || Cq < 1 || Cq > L || iters < 0) {
        set_static_error("ac_cluster_q_noalloc: invalid argument");
        return AC_ERR_INVALID_ARG;
    }
    if (d != 64 && d != 128) {
        set_static_error("ac_cluster_q_noalloc: d must be 64 or 128");
        return AC_ERR_UNSUPPORTED;
    }
    const int64_t rows = (int64_t)BH * L;
    if (rows > kMaxRows || (int64_t)BH * (Cq + 1) > kMaxCentreSlots || Cq > kMaxCq) {
        set_static_error("ac_cluster_q_noalloc: B*H*L must be <= 1048576, B*H*(Cq+1) <= 65536 and Cq <= 4096");
        return AC_ERR_INVALID_ARG;
    }
    void *base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) {
        set_static_error("ac_cluster_q_noalloc: cudaGetSymbolAddress of the scratch array failed");
        return AC_ERR_CUDA;
    }
    unsigned char *sb = static_cast<unsigned char *>(base);
    uint32_t *err = err_out ? err_out : reinterpret_cast<uint32_t *>(sb);
    float *inv = reinterpret_cast<float *>(sb + kErrBytes);
    int *perm = reinterpret_cast<int *>(sb + kErrBytes + kInvBytes);
    int *offs = reinterpret_cast<int *>(sb + kErrBytes + kInvBytes + kPermBytes);
    int *counts = reinterpret_cast<int *>(sb + kErrBytes + kInvBytes + kPermBytes + kOffsBytes);

    cudaStream_t s = (cudaStream_t)stream;
    const bf16 *Qb = reinterpret_cast<const bf16 *>(Q);
    const int64_t cstride = (int64_t)Cq * d;
    // The error word starts at zero; every other scratch word read below is
    // first written in this call (norms, permutation, offsets and counts).
    if ((e = cudaMemsetAsync(err, 0, sizeof(uint32_t), s)) != cudaSuccess) goto cuda_error;
    if ((e = launch_qnorm(Qb, inv, rows, d, err, s)) != cudaSuccess) goto cuda_error;
    if (init_centroids) {
        if (init_centroids != centroids_out &&
            (e = cudaMemcpyAsync(centroids_out, init_centroids, sizeof(float) * BH * cstride,
                                 cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
            goto cuda_error;
    } else {
        SeedArgs sa{Qb, inv, L, nullptr, nullptr, L, centroids_out, cstride, nullptr, nullptr, Cq, Cq, seed, 0, BH, d};
        if ((e = launch_seed(sa, s)) != cudaSuccess) goto cuda_error;
    }
    {
        AssignArgs as{Qb, inv, L, nullptr, nullptr, L, centroids_out, cstride, nullptr, nullptr, Cq, labels_out,
                      nullptr, BH, d};
        SortArgs so{labels_out, L, nullptr, L, nullptr, Cq, Cq, perm, offs, Cq + 1, counts, Cq, BH, nullptr};
        UpdateArgs up{Qb, inv, L, nullptr, perm, offs, Cq + 1, centroids_out, cstride, nullptr, nullptr, Cq, BH, d, Cq};
        up.err = err;
        for (int t = 0; t < iters; ++t) {
            if ((e = launch_assign_exact(as, s)) != cudaSuccess) goto cuda_error;
            if ((e = launch_counting_sort(so, s)) != cudaSuccess) goto cuda_error;
            if ((e = launch_update(up, s)) != cudaSuccess) goto cuda_error;
        }
        if ((e = launch_assign_exact(as, s)) != cudaSuccess) goto cuda_error;
    }
    return AC_OK;
cuda_error:
    set_static_error("ac_cluster_q_noalloc: a kernel launch failed");
    return AC_ERR_CUDA;
}
