/*
 * ac.h -- C ABI of libac, cluster-routed sparse attention for one video-DiT
 * attention layer on one NVIDIA B200 (sm_100a).
 *
 * The method is AdaCluster ("AdaCluster: Adaptive Query-Key Clustering for
 * Sparse Attention in Video Generation", arXiv 2604.18348), Algorithm 3:
 *   line 3   A_q, C_q <- KMeans(Normalize(Q))                 ac_cluster_q
 *   line 4   A_k, C_k, F <- MultiStageClustering(K, tau, N_max)
 *            (Algorithm 1, Sec. 3.2.2)                        ac_cluster_k_multistage
 *   line 8-9 S <- TensorQuest; Index <- argtopk(S, topk)
 *            (Sec. 3.2.3, Eq. (1), Algorithm 2)               ac_score_select
 *   line 5-11 AttnOut <- Attention(Q, K*, V*), dense when F   ac_sparse_attn
 *   all of the above                                          ac_layer_forward
 *
 * Conventions shared by every entry point:
 *  - Tensors are caller-owned and contiguous.  Q, K, V, O are [B, H, L, d]
 *    bf16, passed as uint16_t bit patterns.  d must be 64 or 128.
 *  - "device" pointers must point to memory of the device that was current
 *    at ac_create; "host" pointers to host memory (pinned memory gives
 *    asynchronous copies).  Nullable output pointers may be NULL.
 *  - The library never frees caller memory.  The context owns a workspace
 *    (sized at ac_create from B, H, L, d and the config) and the state that a
 *    warm-started denoising step reuses.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    is asynchronous on that stream, except where noted: the step-0
 *    multi-stage clustering reads back the unabsorbed-set sizes once per
 *    stage and therefore synchronises `stream`.
 *  - Every function returns ac_status.  On error, ac_last_error_string(ctx)
 *    describes it; no C++ exception crosses the ABI.  A context whose kernel
 *    reported an error keeps working for later calls.
 *  - Calls on one context must not overlap (one stream, or serialised).
 */
#ifndef AC_H
#define AC_H

#include <stdint.h>

#if defined(__GNUC__)
#define AC_API __attribute__((visibility("default")))
#else
#define AC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ac_status {
    AC_OK = 0,
    AC_ERR_INVALID_ARG = 1,  /* NULL where not allowed, bad sizes or config   */
    AC_ERR_UNSUPPORTED = 2,  /* d not in {64, 128}, or not an sm_100 device  */
    AC_ERR_WORKSPACE = 3,    /* device allocation failed                      */
    AC_ERR_CUDA = 4,         /* a CUDA runtime call failed                     */
    AC_ERR_NONFINITE = 5,    /* NaN or Inf in an input                          */
    AC_ERR_TIMEOUT = 6,      /* a bounded in-kernel wait expired                */
    AC_ERR_STATE = 7         /* call needs state that is not there (e.g. warm
                                step before any step 0)                        */
} ac_status;

/* Rule for the distance threshold tau of Algorithm 1.  The pages define it as
 * 1.5x the mean token-to-centre distance of the first inference step
 * (Sec. 4.1) and also use absolute thresholds (App. A.5, Table 7).  tau is one
 * number per call, computed from the stage-0 distances of all (batch, head)
 * units together. */
typedef enum ac_tau_mode {
    AC_TAU_ABSOLUTE = 0,     /* tau = tau_value                                */
    AC_TAU_MEAN_FACTOR = 1,  /* tau = tau_value * mean stage-0 distance        */
    AC_TAU_PERCENTILE = 2    /* tau = nearest-rank quantile, tau_value permille */
} ac_tau_mode;

typedef struct ac_config {
    int32_t Cq;          /* query clusters (65 in Sec. 4.1)                        */
    int32_t m0;          /* key clusters of stage 0 of Algorithm 1 ("moderate")   */
    int32_t n_max;       /* N_max of Algorithm 1: cluster count that forces dense */
    int32_t tau_mode;    /* ac_tau_mode                                          */
    float tau_value;     /* see ac_tau_mode                                       */
    int32_t topk;        /* >0: key clusters kept per query cluster;
                            <0: -permille of the head's cluster count (ceil)      */
    int32_t iters_q;     /* Lloyd iterations of the query k-means (step 0)        */
    int32_t iters_k;     /* Lloyd iterations of each key stage (step 0)           */
    int32_t iters_warm;  /* Lloyd iterations of a warm-started step              */
    int32_t stage_rule;  /* cluster count m_t of stages t > 0 of Algorithm 1
                            (line 11, "a moderate cluster number"):
                            0: m_t = min(m0, |U|) (same choice every stage);
                            1: m_t = min(|U|, max(1, ceil(m0 |U| / L)))           */
    uint64_t seed;       /* seeds the initial centres of step 0                   */
    float scale;         /* softmax scale; 0 selects 1/sqrt(d)                    */
    int32_t score_mode;  /* cluster scores before the top-k (Algorithm 3 line 9):
                            0: the Eq. (1) TensorQuest bound (the method);
                            1: mean-based, q . mu with mu the key cluster's centre
                               (the "w/o Quest" ablation of Sec. 4.4, Table 4)    */
    int32_t tail_merge;  /* query-tile tail merging before the attention (iCATS,
                            "tail merging strategy"): 0: off; 1: query clusters
                            that select the same key clusters share tiles
                            (lossless); 2: also, two clusters whose tails are
                            each other's nearest selection (Hamming) and fit one
                            128-row tile pool them: the higher index hands its
                            tail to the lower, which attends to the union      */
    int32_t unit0;       /* (batch, head) index of this context's first unit in
                            the layer, >= 0: unit u of the context seeds its
                            initial centres as unit unit0 + u, so a layer split
                            over contexts (ac_set_tau_exchange) clusters each
                            head as a single context over all heads would; 0
                            for a whole layer                                */
    int32_t compensate;  /* 1: every unselected non-empty key cluster also enters
                            each query's softmax as one pseudo-key, its member
                            mean, weighted by its size (ClusterAttention Sec. 1.2,
                            Eq. (5)-(6)); 0: off.  Not with tail_merge.        */
} ac_config;

typedef struct ac_ctx ac_ctx;

/* Per-stage device time of one ac_layer_forward, in milliseconds, measured with
 * CUDA events on the call's stream. */
typedef struct ac_stage_times {
    float q_cluster_ms;     /* query normalisation + angular k-means            */
    float k_cluster_ms;     /* multi-stage (step 0) or warm key k-means          */
    float stats_sort_ms;    /* key stats and cluster-order permutations          */
    float score_select_ms;  /* Quest scores + top-k + key ranges                  */
    float attention_ms;     /* gathers into cluster order + sparse attention      */
    float attn_kernel_ms;   /* the sparse attention kernel alone                  */
    float total_ms;
} ac_stage_times;

/* Create a context for [B, H, L, d] layers and allocate its workspace.
 * cfg is copied.  Requires B, H, L >= 1; d in {64, 128}; 1 <= Cq <= L and
 * (Cq + 64) * d * 4 <= 200 KiB (Cq <= 336 at d = 128: the query centroids of
 * a head are staged whole in shared memory for Eq. (1)); 1 <= m0 <= L;
 * n_max >= 1; n_max + m0 <= 16384; iteration counts >= 0; an sm_100 device
 * current.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
AC_API ac_status ac_create(const ac_config *cfg, int32_t B, int32_t H, int32_t L, int32_t d,
                    ac_ctx **out);

/* Free the context and its workspace (synchronises the device first). */
AC_API ac_status ac_destroy(ac_ctx *ctx);

/* Last error message of the context; with ctx == NULL, the last error of a
 * context-free call (ac_cluster_q_noalloc) in this thread. */
AC_API const char *ac_last_error_string(const ac_ctx *ctx);

/* Algorithm 3 line 3, Sec. 3.1 / App. A.2: L2-normalise every query (fp32)
 * and run standard k-means with Cq centres on the normalised queries; the
 * centres stay plain means.  Q: device [B,H,L,d] bf16.  init_centroids:
 * nullable device [B,H,Cq,d] fp32 (previous denoising step); NULL seeds the
 * centres from the queries.  iters < 0 selects cfg.iters_q (no init) or
 * cfg.iters_warm (with init).  Outputs (nullable, device): labels_out
 * [B,H,L] int32 in [0,Cq); centroids_out [B,H,Cq,d] fp32.  The state is kept
 * in the context for ac_score_select / ac_sparse_attn. */
AC_API ac_status ac_cluster_q(ac_ctx *ctx, const uint16_t *Q, const float *init_centroids, int32_t iters,
                       int32_t *labels_out, float *centroids_out, void *stream);

/* Algorithm 1 (Sec. 3.2.2) on every (batch, head): stages of k-means on the
 * unabsorbed keys, removal of keys within tau of their centre, dense fallback
 * flag F when the cluster count reaches n_max at a loop head, then the
 * assignment of every key to its closest centre.  Also computes the key
 * cluster statistics (count, per-dimension max/min, SSE) and the compactness
 * Comp = 1/MSE of Sec. 3.2.1.
 * Warm start (Sec. 3.2.2 "Efficient initialization"): when warm_centroids and
 * warm_n_k are non-NULL, the cluster count of each head is kept, the given
 * centres initialise cfg.iters_warm Lloyd iterations over all keys, and heads
 * with warm_dense[h] != 0 stay dense.  All three are device pointers:
 * warm_centroids [B,H,n_max+m0,d] fp32, warm_n_k [B,H] int32, warm_dense
 * [B,H] uint8 (nullable: no dense heads).
 * K: device [B,H,L,d] bf16.  Outputs (nullable, device): labels_out [B,H,L]
 * int32; centroids_out [B,H,n_max+m0,d] fp32; n_k_out [B,H] int32;
 * dense_flag_out [B,H] uint8; comp_out [B,H] fp32.
 * Step 0 synchronises `stream` once per stage. */
AC_API ac_status ac_cluster_k_multistage(ac_ctx *ctx, const uint16_t *K, const float *warm_centroids,
                                  const int32_t *warm_n_k, const uint8_t *warm_dense,
                                  int32_t *labels_out, float *centroids_out, int32_t *n_k_out,
                                  uint8_t *dense_flag_out, float *comp_out, void *stream);

/* Sec. 3.2.3 Eq. (1) and Algorithm 3 line 9, from the state of the two calls
 * above: S[qc,kc] = sum_d max(c_d * Kmax_d, c_d * Kmin_d) with c the query
 * cluster centre, empty key clusters excluded; per query cluster the k best
 * key clusters, ties to the lower id, listed in ascending id order.
 * topk: 0 selects cfg.topk; otherwise as ac_config.topk.  k is clamped to
 * [1, non-empty clusters] per head.  Outputs (nullable, device): sel_out
 * [B,H,Cq,n_max+m0] int32 (first k_out[h] entries of each row valid);
 * k_out [B,H] int32.  Also builds the per-query-cluster key ranges that
 * ac_sparse_attn walks. */
AC_API ac_status ac_score_select(ac_ctx *ctx, int32_t topk, int32_t *sel_out, int32_t *k_out,
                          void *stream);

/* Algorithm 3 lines 5-11: for every query, exact softmax attention (scale
 * cfg.scale, fp32 accumulation) over the keys of the key clusters selected
 * for its query cluster, or over all keys of a dense head.  Q, K, V must be
 * the tensors whose Q and K were clustered by the calls above.  The call first
 * gathers Q, K, V into cluster order (context-owned copies), then runs the
 * attention kernel.  O: device [B,H,L,d] bf16, written in the original token
 * order. */
AC_API ac_status ac_sparse_attn(ac_ctx *ctx, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                         uint16_t *O, void *stream);

/* The whole layer: ac_cluster_q, ac_cluster_k_multistage, ac_score_select and
 * ac_sparse_attn.  warm = 0: step 0 (seeded init, multi-stage keys);
 * warm = 1: a later denoising step that warm-starts from the centres, cluster
 * counts and dense flags the context kept from the previous call (requires
 * one earlier call, else AC_ERR_STATE).  times: nullable; when given, the
 * call synchronises `stream` to fill it. */
AC_API ac_status ac_layer_forward(ac_ctx *ctx, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                           uint16_t *O, int32_t warm, ac_stage_times *times, void *stream);

/* ac_layer_forward from host memory: copies hQ, hK, hV (host [B,H,L,d] bf16)
 * into context-owned device buffers on `stream`, runs the layer, copies O
 * back into hO (host) and synchronises `stream`. */
AC_API ac_status ac_layer_forward_host(ac_ctx *ctx, const uint16_t *hQ, const uint16_t *hK,
                                const uint16_t *hV, uint16_t *hO, int32_t warm, void *stream);

/* ac_layer_forward_host without waiting: enqueues the input copies (on a
 * context-owned copy stream), the layer (on `stream`) and the output copy (on a
 * second copy stream) and returns.  Consecutive calls pipeline: call n's input
 * copy overlaps call n - 1's layer and its output copy call n + 1's layer
 * (two context-owned device staging sets, used alternately); within a call
 * the query clustering starts once Q has landed, while K and V still copy.
 * Ownership: hQ, hK, hV must stay unchanged, and hO must not be read, until
 * the call is complete: after ac_synchronize(ctx, stream) returns, or once
 * `stream` has passed an ac_join(ctx, stream).  Host buffers should be pinned
 * (pageable memory makes the copies synchronous).  Errors: argument and launch
 * errors are returned; errors that kernels record on the device are reported
 * by the next ac_synchronize. */
AC_API ac_status ac_layer_forward_host_async(ac_ctx *ctx, const uint16_t *hQ, const uint16_t *hK,
                                      const uint16_t *hV, uint16_t *hO, int32_t warm, void *stream);

/* Make `stream` wait (without blocking the host) until the output copies of
 * every earlier ac_layer_forward_host_async call have finished. */
AC_API ac_status ac_join(ac_ctx *ctx, void *stream);

/* Wait for the work enqueued on `stream` (and for the output copies of earlier
 * ac_layer_forward_host_async calls) and report any error that a kernel
 * recorded on the device (AC_ERR_TIMEOUT, AC_ERR_NONFINITE); clears it. */
AC_API ac_status ac_synchronize(ac_ctx *ctx, void *stream);

/* Health check of the failure-detection path.  Launches on `stream` one CTA
 * whose thread waits, with the same bounded loop (globaltimer, clock64 and a
 * poll count) that the pipelined kernels use on their mbarriers, for a phase
 * that never completes, with a time limit of limit_us microseconds
 * (1 .. 2,000,000).  When the limit runs out the kernel records the timeout in
 * the context's device error word and returns, so the next ac_synchronize
 * reports AC_ERR_TIMEOUT (and clears it) and the context stays usable.
 * Errors: AC_ERR_INVALID_ARG for a NULL context or a limit out of range;
 * AC_ERR_CUDA when the launch fails. */
AC_API ac_status ac_check_wait_timeout(ac_ctx *ctx, int32_t limit_us, void *stream);

/* Read-only views of intermediate device tensors (for tests and metrics).
 * *dev_ptr receives a device pointer owned by the context, shape[0..3] the
 * extents (unused trailing extents are 1).  Contents are valid after the
 * producing call has completed on its stream. */
typedef enum ac_tensor_id {
    AC_T_INV_NORM_Q = 0,   /* fp32  [BH, L]            1/||q||                */
    AC_T_LABELS_Q = 1,     /* int32 [BH, L]                                     */
    AC_T_CENT_Q = 2,       /* fp32  [BH, Cq, d]                                 */
    AC_T_COUNTS_Q = 3,     /* int32 [BH, Cq]                                    */
    AC_T_PERM_Q = 4,       /* int32 [BH, L]   token at each cluster-order slot   */
    AC_T_OFFS_Q = 5,       /* int32 [BH, Cq+1]                                  */
    AC_T_LABELS_K = 6,     /* int32 [BH, L]                                     */
    AC_T_DMIN_K = 7,       /* fp32  [BH, L]   squared distance to own centre    */
    AC_T_CENT_K = 8,       /* fp32  [BH, Ccap, d]  Ccap = n_max + m0            */
    AC_T_N_K = 9,          /* int32 [BH]                                        */
    AC_T_DENSE = 10,       /* uint8 [BH]                                        */
    AC_T_COUNTS_K = 11,    /* int32 [BH, Ccap]                                  */
    AC_T_KMAX = 12,        /* bf16  [BH, Ccap, d]                               */
    AC_T_KMIN = 13,        /* bf16  [BH, Ccap, d]                               */
    AC_T_SSE = 14,         /* fp32  [BH, Ccap]                                  */
    AC_T_COMP = 15,        /* fp32  [BH]                                        */
    AC_T_PERM_K = 16,      /* int32 [BH, L]                                     */
    AC_T_OFFS_K = 17,      /* int32 [BH, Ccap+1]                                */
    AC_T_SCORE = 18,       /* fp32  [BH, Cq, Ccap]                              */
    AC_T_SEL = 19,         /* int32 [BH, Cq, Ccap]                              */
    AC_T_KSEL = 20,        /* int32 [BH]                                        */
    AC_T_TAU = 21,         /* fp32  [1]                                         */
    AC_T_STAGES = 22,      /* int32 [BH]   stages run by Algorithm 1            */
    AC_T_REMOVED_STAGE = 23, /* int32 [BH, L] stage that absorbed the key, -1 */
    AC_T_MSE = 24,         /* fp32  [BH]                                        */
    AC_T_FALLBACK_AT = 25, /* int32 [BH]   after step 0: the largest n_max under
                              which the unit would have fallen back to dense
                              attention (the cluster count at the head of its
                              last stage; 0 when stage 0 absorbed every key; for
                              a unit that fell back, its count then)         */
    AC_T_NUM = 26
} ac_tensor_id;

AC_API ac_status ac_get_tensor(ac_ctx *ctx, int32_t which, void **dev_ptr, int64_t shape[4]);

/* Work counters of the last ac_sparse_attn (synchronises the device):
 * kept key tokens summed over queries, the same in computed (padded) tile
 * columns, the number of work items (pairs of 128-query tiles), dense units,
 * and the location of the first in-kernel wait that gave up (0 if none). */
typedef struct ac_attn_counters {
    int64_t kept_pairs;       /* sum over queries of |K*|                        */
    int64_t computed_pairs;   /* sum over tiles of 128 x computed key columns   */
    int64_t tiles;
    int64_t dense_heads;
    int64_t wait_failure;     /* 0, or where the first bounded wait gave up:
                                 1<<60 | role<<24 | barrier<<16 | tile<<1 | parity */
} ac_attn_counters;

AC_API ac_status ac_get_attn_counters(ac_ctx *ctx, ac_attn_counters *out);

/* Diagnostics of the k-means assignments since the context was created (or
 * last reset).  The assignments of Sec. 3.1 and of Algorithm 1 (stage 0, the
 * final pass over all of C) and of the warm-started Lloyd passes run on the
 * tensor cores: centres split into bf16 + remainder, x . c_hi per pair, then
 * a rigorous error bound decides each row; rows the bound cannot settle are
 * rescored with the exact fp32 arithmetic, so labels equal the exact
 * definition's.  Stages t >= 1 of Algorithm 1 run on a gathered copy of the
 * unabsorbed keys, on the tensor cores too; only inputs that are not 16-byte
 * aligned take the exact CUDA-core kernel.  The environment variable
 * AC_EXACT_ASSIGN=1 at ac_create forces the exact kernel everywhere.
 * Synchronises `ctx`'s device; reset != 0 zeroes the counters afterwards. */
typedef struct ac_assign_counters {
    int64_t tensor_passes;      /* assignment passes run on the tensor cores   */
    int64_t exact_passes;       /* assignment passes run by the exact kernel   */
    int64_t rows;               /* rows assigned by the tensor-core passes     */
    int64_t uncertain_rows;     /* of those, rescored exactly (candidates)     */
    int64_t full_rescore_rows;  /* of those, rescored against every centre     */
} ac_assign_counters;

AC_API ac_status ac_get_assign_counters(ac_ctx *ctx, ac_assign_counters *out, int32_t reset);

/* The query clustering of ac_cluster_q (normalise, then Lloyd k-means with
 * Cq centres) without a context and without allocating device memory.  The
 * paper has no counterpart of this entry point; it exists for callers that
 * cannot call cudaMalloc while they run: a plugin's enqueue callback inside an
 * inference engine, a server that must not grow its footprint while serving,
 * or a process whose device memory belongs to another allocator.
 *  - Q: device [BH, L, d] bf16 (d in {64, 128}).  init_centroids: nullable
 *    device [BH, Cq, d] fp32 (NULL: seeded from the queries with `seed`, as
 *    ac_cluster_q does).  iters >= 0 Lloyd iterations, then a final assignment.
 *  - Outputs (device, required): labels_out [BH, L] int32; centroids_out
 *    [BH, Cq, d] fp32, also used as the working centres (updated in place).
 *  - err_out: nullable device uint32.  The call sets it to 0 on `stream`, and
 *    its kernels OR in their error bits: 1 = a bounded in-kernel wait expired
 *    (the outputs are not valid), 4 = NaN or Inf in Q.  Read it once `stream`
 *    has passed the call.  With NULL, errors are recorded in the scratch array
 *    and cannot be read.
 *  - Limits: BH*L <= 1048576, BH*(Cq+1) <= 65536 and Cq <= 4096 (the sort's
 *    shared-memory histograms), else AC_ERR_INVALID_ARG before any work.  The
 *    scratch (error word, norms, permutation, offsets, counts) is one 8.5 MiB
 *    __device__ array that every GPU which loads libac holds until the process
 *    exits; nothing is allocated per call.
 *  - The first call in a CUDA context looks the array's address up
 *    (cudaGetSymbolAddress) and keeps it per context, so a context that was
 *    reset and created again looks it up anew; make the first call in a
 *    context before any stream capture.
 *  - Every call shares the one array: calls that overlap on the GPU (two
 *    streams, two threads) race and corrupt each other's results.  Serialise
 *    them.  Asynchronous on `stream`. */
AC_API ac_status ac_cluster_q_noalloc(const uint16_t *Q, int32_t BH, int32_t L, int32_t d, int32_t Cq,
                                      int32_t iters, uint64_t seed, const float *init_centroids,
                                      int32_t *labels_out, float *centroids_out, uint32_t *err_out,
                                      void *stream);

/* Splitting the heads of one layer over several contexts (one per GPU or
 * rank; Algorithm 1 works per (batch, head), the only coupling of the heads is
 * tau, pooled over the stage-0 distances of every head of the layer, Sec. 4.1).
 * With an exchange function set, the step-0 key clustering of the context
 * reduces its own heads' stage-0 distances and calls fn(user, data, count) on
 * the calling thread: data (host memory) holds `count` partial sums that fn
 * must replace, in place, by their sums over all contexts of the layer (for
 * example an all-reduce over the ranks), returning 0 on success.  The calls
 * are, in order, for the mean rule: count 2, {sum over the distances d_i of
 * floor(d_i 2^24), number of distances}; for the percentile rule: count 1, the
 * number of distances, then four times count 256, the histogram of the next
 * 8-bit digit of the distances' bit patterns among those that match the digits
 * chosen so far (radix select, most significant digit first).  Every context
 * of the layer must take part in the same step-0 calls.  The absolute rule
 * exchanges nothing.  The pooled tau equals the one a single context over all
 * heads computes, bit for bit.  fn = NULL: tau from this context's heads.
 * Errors: INVALID_ARG; the step-0 call returns AC_ERR_STATE if fn fails. */
typedef int32_t (*ac_sum_u64_fn)(void *user, uint64_t *data, int32_t count);
AC_API ac_status ac_set_tau_exchange(ac_ctx *ctx, ac_sum_u64_fn fn, void *user);

/* Host-side steps of the pooled tau (no device work; used by the step-0
 * clustering when an exchange function is set, and callable on their own).
 * ac_tau_mean_from_sums: tau = factor * ((fixed_sum / 2^24) / n), in fp64
 * rounded to nearest, then to fp32 (Sec. 4.1, 1.5x the mean stage-0
 * distance).  ac_tau_radix_pick: one digit of a nearest-rank selection:
 * state = {prefix, mask, rank}; given the summed 256-bin histogram of the
 * digit at `shift` (24, 16, 8, 0) among the distances whose bits match
 * prefix under mask, it appends the digit that holds the rank-th smallest
 * (0-based) distance and leaves the rank within that digit; after the pass
 * with shift 0, prefix is the bit pattern of the selected distance.
 * Errors: INVALID_ARG (n = 0, bad shift, or a histogram with fewer entries than
 * rank + 1). */
AC_API ac_status ac_tau_mean_from_sums(float factor, uint64_t fixed_sum, uint64_t n, float *tau);
AC_API ac_status ac_tau_radix_pick(const uint64_t *hist, int32_t shift, uint32_t *state);

/* Calibration of N_max over a stack of layers (AdaCluster Sec. 4.1: k_max is
 * set so that the top 15% of layers, the least compact ones, run full
 * attention).  Given each unit's AC_T_FALLBACK_AT from a step 0 run with an
 * n_max large enough that no unit fell back, returns in *n_max the n_max
 * under which the ceil(dense_frac * n) units with the largest values fall
 * back: the k-th largest value (units tied with it fall back too).  When fewer
 * than k units ran more than one stage, *n_max is the smallest positive value
 * (only the multi-stage units can fall back), or n_max = 1 + max when
 * dense_frac is 0.  Host only.  Errors: INVALID_ARG (n < 1, dense_frac outside
 * [0, 1], or no unit ran more than one stage while dense_frac > 0). */
AC_API ac_status ac_calibrate_n_max(const int32_t *fallback_at, int64_t n, float dense_frac, int32_t *n_max);

/* Number of kernels libac has launched in this process so far (all contexts). */
AC_API ac_status ac_get_launch_count(int64_t *out);

/* Warm-start state (query centres, key centres, cluster counts, dense flags)
 * to and from host memory, for checkpoint / resume across denoising steps.
 * ac_state_export with host_buf == NULL stores the needed size in *bytes.
 * Both synchronise the device. */
AC_API ac_status ac_state_export(ac_ctx *ctx, void *host_buf, int64_t *bytes);
AC_API ac_status ac_state_import(ac_ctx *ctx, const void *host_buf, int64_t bytes);

#ifdef __cplusplus
}
#endif

#endif /* AC_H */
