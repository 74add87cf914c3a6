// noalloc.cu -- query clustering for callers that cannot allocate device memory.
//
// ac_cluster_q_noalloc does the work of ac_cluster_q (L2-normalise the
// queries, then Lloyd k-means on the unit vectors) without a context and
// without any device allocation.  Its scratch -- the inverse query norms, the
// cluster-order permutation and the per-cluster offsets and counts -- lives in
// one file-scope __device__ array of fixed size, which every GPU that loads
// libac holds until the process exits.  The caller supplies only the inputs and
// the outputs (labels and centres; the centres are updated in place).
//
// Who needs this: code that runs where cudaMalloc is not allowed or not wise --
// inside a plugin's enqueue callback of an inference engine, in a server that
// must not grow its memory footprint while serving, or in a process whose
// device memory is entirely owned by another allocator.
#include <mutex>

#include "ac_device.cuh"
#include "ac_internal.h"

namespace {

constexpr int64_t kMaxRows = int64_t(1) << 20;  // B*H*L
constexpr int64_t kMaxCentreSlots = 1 << 16;    // B*H*(Cq+1)

constexpr size_t kInvBytes = sizeof(float) * kMaxRows;
constexpr size_t kPermBytes = sizeof(int) * kMaxRows;
constexpr size_t kOffsBytes = sizeof(int) * kMaxCentreSlots;
constexpr size_t kCountBytes = sizeof(int) * kMaxCentreSlots;
constexpr size_t kScratchBytes = kInvBytes + kPermBytes + kOffsBytes + kCountBytes;  // 8.5 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device.
std::mutex g_mu;
void *g_addr[256] = {};

cudaError_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace

using namespace ac;

extern "C" ac_status ac_cluster_q_noalloc(const uint16_t *Q, int32_t BH, int32_t L, int32_t d, int32_t Cq,
                                          int32_t iters, uint64_t seed, const float *init_centroids,
                                          int32_t *labels_out, float *centroids_out, void *stream) {
    if (!Q || !labels_out || !centroids_out || BH < 1 || L < 1 || Cq < 1 || Cq > L || iters < 0) {
        set_static_error("ac_cluster_q_noalloc: invalid argument");
        return AC_ERR_INVALID_ARG;
    }
    if (d != 64 && d != 128) {
        set_static_error("ac_cluster_q_noalloc: d must be 64 or 128");
        return AC_ERR_UNSUPPORTED;
    }
    const int64_t rows = (int64_t)BH * L;
    if (rows > kMaxRows || (int64_t)BH * (Cq + 1) > kMaxCentreSlots) {
        set_static_error("ac_cluster_q_noalloc: B*H*L must be <= 1048576 and B*H*(Cq+1) <= 65536");
        return AC_ERR_INVALID_ARG;
    }
    void *base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) {
        set_static_error("ac_cluster_q_noalloc: cudaGetSymbolAddress of the scratch array failed");
        return AC_ERR_CUDA;
    }
    unsigned char *sb = static_cast<unsigned char *>(base);
    float *inv = reinterpret_cast<float *>(sb);
    int *perm = reinterpret_cast<int *>(sb + kInvBytes);
    int *offs = reinterpret_cast<int *>(sb + kInvBytes + kPermBytes);
    int *counts = reinterpret_cast<int *>(sb + kInvBytes + kPermBytes + kOffsBytes);

    cudaStream_t s = (cudaStream_t)stream;
    const bf16 *Qb = reinterpret_cast<const bf16 *>(Q);
    const int64_t cstride = (int64_t)Cq * d;
    // Every scratch word read below is first written in this call (norms,
    // permutation, offsets and counts), so nothing needs clearing.
    if ((e = launch_qnorm(Qb, inv, rows, d, nullptr, s)) != cudaSuccess) goto cuda_error;
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
