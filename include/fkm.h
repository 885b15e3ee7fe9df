/*
 * fkm.h -- C ABI of libfkm: exact batched Lloyd k-means on NVIDIA B200 (sm_100a).
 *
 * The problem is the one the Flash-KMeans pages state with
 * batch_kmeans_Euclid(x, n_clusters, max_iters, tol) -> (cluster_ids, centers, _)
 * ("Flash-KMeans" GitHub README, section "Usage"): B independent problems, each
 * N points of dimension D clustered into K centroids by Lloyd iterations
 * (assign every point to its nearest centroid, then move every centroid to the
 * mean of its points), minimising sum_i ||x_i - c_{a_i}||^2 ("Flash-KMeans：快速且
 * 内存高效精确K-Means聚类" summary, section 前置知识 / K-Means聚类算法).
 *
 * Conventions shared by every entry point
 *   Layout     x is [B, N, D] row-major and contiguous, in `dtype`.
 *              Centroids are float32 [B, K, D]; ids int32 [B, N] (values in
 *              [0, K)); counts int32 [B, K]; per-batch scalars are [B].
 *   Pointers   "device" = memory the current CUDA device can address (cudaMalloc
 *              or torch CUDA tensors); "host" = CPU memory.  Every pointer must
 *              be 16-byte aligned.  The caller owns every buffer; the library
 *              allocates no device memory of its own: scratch comes from the
 *              caller's workspace (see fkm_workspace_size), whose size never
 *              depends on N*K (the B x N x K distance matrix is never formed).
 *   Streams    `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *              stream).  Work is stream-ordered; functions marked "async" return
 *              before the GPU finishes.  The library's kernels are launched as
 *              programmatic dependents (each waits for the stream's previous
 *              work to complete before it touches memory) and let the next
 *              kernel be scheduled early: a caller kernel launched after a call
 *              with programmatic stream serialization of its own must wait
 *              (griddepcontrol.wait) before it reads the call's outputs; an
 *              ordinary launch is ordered as usual.
 *   Limits     B, N, K, D >= 1; D * sizeof(dtype) a multiple of 16 bytes
 *              (D % 8 == 0 for bf16/fp16, D % 4 == 0 for fp32);
 *              D <= 4096; B*N < 2^31; B*K < 2^31.  Above D = 256 (fp32:
 *              128) the assign kernel streams the point tile in 64-column
 *              chunks and the update sums 512-byte column slabs.
 *   Errors     Arguments are validated before anything is launched; a violation
 *              returns FKM_ERR_INVALID_ARG or FKM_ERR_UNSUPPORTED and launches
 *              nothing.  There is no fallback path of any kind.  CUDA failures
 *              return FKM_ERR_CUDA.  Kernels report what they detect (a bounded
 *              wait that ran out, an out-of-range id) in a status word inside
 *              the workspace, read by fkm_sync_status (and by fkm_lloyd itself).
 *              fkm_last_error() gives a thread-local description of the last
 *              failure.
 */
#ifndef FKM_H_
#define FKM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FKM_API __attribute__((visibility("default")))
#else
#define FKM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FKM_OK = 0,
  FKM_ERR_INVALID_ARG = 1,
  FKM_ERR_UNSUPPORTED = 2,
  FKM_ERR_CUDA = 3,
  FKM_ERR_WORKSPACE_TOO_SMALL = 4,
  FKM_ERR_TIMEOUT = 5,
  FKM_ERR_INTERNAL = 6,
  FKM_ERR_BAD_ID = 7
} fkm_status;

/* storage type of the points */
typedef enum { FKM_F32 = 0, FKM_F16 = 1, FKM_BF16 = 2 } fkm_dtype;

/* The similarity a run clusters by (fkm_assign_metric, fkm_update_metric,
 * fkm_lloyd_metric; the calls without the suffix are Euclidean).  The README
 * lists cosine and dot-product k-means beside the Euclidean one ("Flash-KMeans"
 * GitHub README, section "Usage", the CuTe backend note) without defining
 * them; the plain readings are taken:
 *   FKM_METRIC_EUCLID   nearest centroid, c_k = mean of its points
 *   FKM_METRIC_DOT      a_i = argmax_k x_i . c_k, c_k = mean of its points,
 *                       objective sum_i x_i . c_{a_i}
 *   FKM_METRIC_COSINE   a_i = argmax_k x_i . c_k / ||c_k||, c_k = s_k / ||s_k||
 *                       (unit direction of its points' sum s_k; spherical
 *                       k-means), objective sum_i x_i . c_{a_i} / ||c_{a_i}||
 * Ties go to the lowest index; an empty cluster, or one whose sum is zero,
 * keeps its previous centroid. */
typedef enum { FKM_METRIC_EUCLID = 0, FKM_METRIC_DOT = 1, FKM_METRIC_COSINE = 2 } fkm_metric;

/* Bytes of device workspace fkm_assign / fkm_update / fkm_lloyd need for this
 * shape (one size serves all three).  Host-only: makes no CUDA call.
 * Returns FKM_ERR_INVALID_ARG / FKM_ERR_UNSUPPORTED for shapes the library
 * rejects.  `bytes` (host) receives the size. */
FKM_API fkm_status fkm_workspace_size(int B, int N, int K, int D, int dtype, size_t* bytes);

/* Assign step (predict): ids[b,i] = argmin_k ||x[b,i] - c_hat[b,k]||^2, ties to
 * the lowest k, where c_hat = m_b + q(c - m_b): m_b is the batch's mean
 * centroid (fp64 sum over k in index order / K, rounded to fp32) and q() the
 * RNE rounding of the fp32 offset c - m_b to `dtype` -- the tensor-core
 * operand.  Centring keeps the products small, so data far from the origin
 * keeps its precision; k-means is translation invariant ("Flash-KMeans"
 * README, section "Centre your data").  For fp32 points the offset is carried
 * in split bf16 hi+lo form (relative error about 2^-17) and c_hat ~= c.
 * Computed as the online argmin of the score over centroid tiles on tcgen05
 * tensor cores, without ever writing a distance matrix ("Flash-KMeans: Fast
 * and Memory-Efficient Exact K-Means" summary, section "Method", FlashAssign;
 * "Flash-KMeans：快速且内存高效精确K-Means聚类" summary, section 方法步骤详情
 * step (1)).
 *   x        device [B,N,D] dtype        centers  device [B,K,D] float32
 *   ids      device [B,N] int32 (out)
 *   inertia  device [B] float64 (out) = sum_i ||x_i - c_hat[b, ids_i]||^2 (direct
 *            difference, fp32 terms summed in fp64), or NULL; with inertia,
 *            B <= 65535 (FKM_ERR_UNSUPPORTED above)
 *   ws       device workspace of ws_bytes >= fkm_workspace_size(...)
 * Async. */
FKM_API fkm_status fkm_assign(int B, int N, int K, int D, int dtype, const void* x, const float* centers,
                      int32_t* ids, double* inertia, void* ws, size_t ws_bytes, void* stream);

/* Update step (sort-inverse update): stable radix argsort of the 1-D ids, one
 * pass over contiguous runs of equal ids gathering rows of the UNPERMUTED x by
 * the sorted index, fp64 sums per run, one flush per run per 512-row range of
 * the sorted order ("Flash-KMeans: Fast and Memory-Efficient Exact K-Means"
 * summary, section "Method", Sort-Inverse Update; "Flash-KMeans：快速且内存高效
 * 精确K-Means聚类" summary, section 方法步骤详情 step (2)).
 *   counts[b,k]   = number of i with ids[b,i] == k (exact)
 *   centers[b,k]  = mean of those x_i (fp64 sum, rounded to fp32), or
 *                   prev_centers[b,k] unchanged when counts[b,k] == 0
 *   shift[b]      = sum_k ||centers[b,k] - prev_centers[b,k]||^2 (float64), or NULL
 *   inertia[b]    = sum_i ||x_i - c_hat[b, ids_i]||^2 (float64), the objective of
 *                   the given assignment against the centroids an assign step
 *                   would have used (c_hat of prev_centers, as in fkm_assign),
 *                   or NULL
 *   x device [B,N,D] dtype; ids device [B,N] int32; prev_centers device [B,K,D];
 *   centers device [B,K,D] (out, must not alias prev_centers); counts device
 *   [B,K] int32 (out).  An id outside [0,K) sets FKM_ERR_BAD_ID in the status
 *   word (rows with such ids are ignored).  Async. */
FKM_API fkm_status fkm_update(int B, int N, int K, int D, int dtype, const void* x,
                              const int32_t* ids, const float* prev_centers, float* centers,
                              int32_t* counts, double* shift, double* inertia, void* ws,
                              size_t ws_bytes, void* stream);

/* Full Lloyd run (batch_kmeans_Euclid).  Starting from init_centers, for
 * t < max_iters: assign, then update; stop after an update when
 * max_b shift[b] < tol (strict, so tol = 0 runs max_iters iterations).
 *   ids      device [B,N] (out): the last assignment
 *   centers  device [B,K,D] (out): the centroids after the last update
 *   counts   device [B,K] (out): sizes of the last assignment's clusters
 *   inertia  device [B] float64 (out): objective of the last assignment against
 *            the centroids it was made with (direct difference), or NULL
 *   n_iter   host int (out): iterations run
 * init_centers may alias centers.  With tol == 0 the iterations are replayed
 * from one captured CUDA graph; with tol > 0 one 8-byte device-to-host read
 * per iteration decides whether to stop.  Synchronous: returns after the
 * stream has finished, with the status word checked. */
FKM_API fkm_status fkm_lloyd(int B, int N, int K, int D, int dtype, const void* x,
                     const float* init_centers, int max_iters, float tol, int32_t* ids,
                     float* centers, int32_t* counts, double* inertia, int* n_iter, void* ws,
                     size_t ws_bytes, void* stream);

/* Dot-product and cosine k-means (fkm_metric above), with the same shapes,
 * layouts, workspace (fkm_workspace_size), validation and stream behaviour
 * as fkm_assign / fkm_update / fkm_lloyd; metric FKM_METRIC_EUCLID gives
 * exactly those calls (without fkm_assign's optional objective).
 *   assign   ids = argmax_k x . c_hat_k over the tensor-core operands
 *            c_hat = m + q(v - m), v = c (dot) or fp32(c / ||c||) (cosine),
 *            m the mean of the v rows; x . m is the same for every k, so the
 *            bias product is zero and the epilogue compares x . q(v - m).
 *   update   centers = the mean of each cluster's points (dot), or its unit
 *            direction (cosine); empty or zero-sum clusters keep prev.
 *            objective [B] (may be NULL) = sum_i x_i . c~_{ids_i}, c~ = prev or
 *            prev / ||prev||: the objective of the assignment, formed from the
 *            cluster sums.  shift as in fkm_update.
 *   lloyd    the loop of the two; objective [B] is that of the last
 *            assignment, against the centroids it used; tol compares the
 *            centroid shift as in fkm_lloyd.
 * An unknown metric returns FKM_ERR_INVALID_ARG before any launch. */
FKM_API fkm_status fkm_assign_metric(int B, int N, int K, int D, int dtype, int metric,
                                     const void* x, const float* centers, int32_t* ids, void* ws,
                                     size_t ws_bytes, void* stream);
FKM_API fkm_status fkm_update_metric(int B, int N, int K, int D, int dtype, int metric,
                                     const void* x, const int32_t* ids, const float* prev_centers,
                                     float* centers, int32_t* counts, double* shift,
                                     double* objective, void* ws, size_t ws_bytes, void* stream);
FKM_API fkm_status fkm_lloyd_metric(int B, int N, int K, int D, int dtype, int metric,
                                    const void* x, const float* init_centers, int max_iters,
                                    float tol, int32_t* ids, float* centers, int32_t* counts,
                                    double* objective, int* n_iter, void* ws, size_t ws_bytes,
                                    void* stream);

/* Device workspace for fkm_lloyd_host with chunks of `chunk_rows` points. */
FKM_API fkm_status fkm_host_workspace_size(int B, int N, int K, int D, int dtype, int64_t chunk_rows,
                                   size_t* bytes);

/* Out-of-core Lloyd run: x stays in HOST memory (pinned, page-locked, e.g.
 * cudaHostAlloc) and is streamed to the device in chunks of chunk_rows points
 * through two device buffers: a copy stream fills one buffer (cudaMemcpyAsync)
 * while the compute stream runs assign + chunk-local update on the other
 * ("Flash-KMeans" GitHub README, section "Large tensor Benchmark"; "Flash-KMeans：
 * 快速且内存高效精确K-Means聚类" summary, section 方法步骤详情 step (3)).
 * Results are the same as fkm_lloyd's.  Outputs (ids, centers, counts,
 * inertia) are device pointers as in fkm_lloyd; x_host is a host pointer.
 * Synchronous.  For failure-detection tests, the environment variable
 * FKM_FAULT_INJECT=h2d@chunk:<n> makes the copy of the n-th streamed chunk
 * fail (FKM_ERR_CUDA) on the host before it is issued; the call then returns
 * with its copy stream and events released. */
FKM_API fkm_status fkm_lloyd_host(int B, int N, int K, int D, int dtype, const void* x_host,
                          const float* init_centers, int max_iters, float tol,
                          int64_t chunk_rows, int32_t* ids, float* centers, int32_t* counts,
                          double* inertia, int* n_iter, void* ws, size_t ws_bytes, void* stream);

/* fkm_lloyd_host under a metric (fkm_metric): dot-product or cosine k-means
 * with the host-streamed points, the same arithmetic as fkm_lloyd_metric
 * (the README lists the metrics beside the Euclidean one; the pages stream
 * host data for any run, "Large tensor Benchmark").  Every chunk's segment
 * sums go to fp64 accumulators, and one finalize per iteration forms the new
 * centroids, the shift and the objective [B] (may be NULL: the objective of
 * the last assignment, against the centroids it used) from them.  Same
 * workspace (fkm_host_workspace_size), validation and synchronisation as
 * fkm_lloyd_host; FKM_METRIC_EUCLID gives exactly fkm_lloyd_host.  An
 * unknown metric returns FKM_ERR_INVALID_ARG before any launch. */
FKM_API fkm_status fkm_lloyd_host_metric(int B, int N, int K, int D, int dtype, int metric,
                                         const void* x_host, const float* init_centers,
                                         int max_iters, float tol, int64_t chunk_rows,
                                         int32_t* ids, float* centers, int32_t* counts,
                                         double* objective, int* n_iter, void* ws,
                                         size_t ws_bytes, void* stream);

/* Stable argsort of n int32 keys in [0, n_keys) on the device (the sort inside
 * fkm_update, exposed for tests): idx[r] = index of the r-th smallest key,
 * equal keys in index order ("Flash-KMeans：快速且内存高效精确K-Means聚类" summary,
 * section 前置知识 / argsort与分段规约, example [3,1,2,1,3,2] -> [1,3,2,5,0,4]).
 * keys, idx: device int32 [n]; workspace from fkm_argsort_workspace_size.
 * n_keys <= 2048 takes the one-pass counting sort that fkm_update and
 * fkm_lloyd use for K <= 2048; larger key ranges take the LSD radix sort
 * (8-bit digits) used for larger K.  A key outside [0, n_keys) sorts after
 * every valid key and sets FKM_ERR_BAD_ID in the status word.  Async. */
FKM_API fkm_status fkm_argsort_workspace_size(int64_t n, int n_keys, size_t* bytes);
FKM_API fkm_status fkm_argsort(const int32_t* keys, int64_t n, int n_keys, int32_t* idx,
                       int32_t* sorted_keys, void* ws, size_t ws_bytes, void* stream);

/* Data-parallel Lloyd over several GPUs ("Flash-KMeans" GitHub README,
 * section "Multi-GPU Support"): the N points of every problem are split into
 * contiguous shards, one per GPU.  One iteration on each GPU is
 *   fkm_assign(shard, c)                        -> shard ids
 *   fkm_partial_update(shard, ids, c)           -> += shard sums / counts / objective
 *   all-reduce of sums, counts and objective across the GPUs (the caller's;
 *   all three are fp64, so one buffer holding them takes one all-reduce)
 *   fkm_finalize_sums(reduced sums, counts, c)  -> the same new centroids everywhere
 *
 * fkm_partial_update: for the shard x [B, N, D] (this GPU's N points of each
 * problem) and its ids [B, N], ADDS the per-cluster fp64 sums of the points
 * to sums [B, K, D] (double), their counts to counts [B, K] (double: exact
 * integers up to 2^53), and, when obj is non-null, the shard's objective
 * sum ||x - c_hat||^2 against the centroids prev [B, K, D] the ids were
 * assigned with to obj [B] (double).  The caller zeroes sums / counts / obj
 * once per iteration.  ws: a workspace of fkm_workspace_size(B, N, K, D,
 * dtype) bytes.  All device pointers, 16-byte aligned.  An id outside
 * [0, K) sets FKM_ERR_BAD_ID in the status word.  Async.
 *
 * fkm_finalize_sums: centers = sums / counts per cluster (IEEE division in
 * fp64, rounded to fp32), prev for a cluster with no points; counts_out
 * [B, K] int32 (may be NULL) receives the counts; shift [B] (may be NULL) =
 * sum_k ||centers - prev||^2.  sums and counts are not modified.  ws: device
 * scratch of at least 256 + 8 * B * K bytes.  centers must not alias prev.
 * Async. */
FKM_API fkm_status fkm_partial_update(int B, int N, int K, int D, int dtype, const void* x,
                                      const int32_t* ids, const float* prev, double* sums,
                                      double* counts, double* obj, void* ws, size_t ws_bytes,
                                      void* stream);
FKM_API fkm_status fkm_finalize_sums(int B, int K, int D, const double* sums,
                                     const double* counts, const float* prev, float* centers,
                                     int32_t* counts_out, double* shift, void* ws,
                                     size_t ws_bytes, void* stream);

/* fkm_partial_update_host: the same shard step for a shard that stays in HOST
 * memory (pinned), as fkm_lloyd_host streams it: each chunk of chunk_rows
 * points is copied to the device, assigned against centers [B, K, D] (fp32,
 * device) and folded into sums / counts / obj exactly as fkm_partial_update
 * adds them; ids [B, N] (device) receive the shard's assignments.  ws: a
 * workspace of fkm_host_workspace_size(B, N, K, D, dtype, chunk_rows) bytes.
 * sums, counts, obj as in fkm_partial_update (the caller zeroes them once per
 * iteration; obj may be NULL).  Synchronous, like fkm_lloyd_host, and
 * FKM_FAULT_INJECT applies to its chunk copies in the same way.
 * flags: 0, or FKM_HOST_COPY_AT_ONCE when no work still queued on `stream`
 * touches this workspace (true after an earlier host-streamed call on it,
 * which synchronises before returning): the first chunk's copy then starts
 * at once instead of after that queued work, so in a data-parallel loop it
 * overlaps the previous iteration's all-reduce and finalize (README
 * "Multi-GPU Support": the first block of the next iteration is prefetched
 * during the all-reduce).  Without the flag the copies wait for the stream. */
#define FKM_HOST_COPY_AT_ONCE 1
FKM_API fkm_status fkm_partial_update_host(int B, int N, int K, int D, int dtype,
                                           const void* x_host, const float* centers,
                                           int64_t chunk_rows, int32_t* ids, double* sums,
                                           double* counts, double* obj, int flags, void* ws,
                                           size_t ws_bytes, void* stream);

/* Centring ("Flash-KMeans" GitHub README, section "Centre your data"):
 * k-means is translation invariant, so points with a large common offset can
 * be clustered after subtracting their mean and the centroids shifted back
 * by it; the tensor-core products then keep their precision.
 *   mu[b, d]      = fp32((sum over i of x[b, i, d], in fp64) / N)
 *   x_out[b,i,d]  = x[b,i,d] - mu[b,d], one fp32 subtraction rounded RNE
 *                   to `dtype` (x_out may be x: centring in place)
 * x, x_out: device [B, N, D] in dtype; mu: device float32 [B, D]; ws: device
 * scratch of fkm_centre_workspace_size bytes.  Limits as for fkm_assign
 * (D * element size a multiple of 16, B * N < 2^31), and B <= 65535
 * (FKM_ERR_UNSUPPORTED above).  Async. */
FKM_API fkm_status fkm_centre_workspace_size(int B, int N, int D, size_t* bytes);
FKM_API fkm_status fkm_centre(int B, int N, int D, int dtype, const void* x, float* mu,
                              void* x_out, void* ws, size_t ws_bytes, void* stream);

/* The centroid side of the same recipe ("Flash-KMeans" GitHub README, section
 * "Centre your data": cluster the centred points, then shift the centroids
 * back by the mean): out[b,k,d] = fp32(centers[b,k,d] + sign * mu[b,d]), one
 * IEEE fp32 addition (sign = +1, back to the original frame) or subtraction
 * (sign = -1, initial centroids into the centred frame) per element.
 * centers, out: device float32 [B, K, D] (out may be centers); mu: device
 * float32 [B, D].  Async on `stream`. */
FKM_API fkm_status fkm_shift_centroids(int B, int K, int D, const float* centers,
                                       const float* mu, int sign, float* out, void* stream);

/* Comparison point, NOT the method: the "standard" iteration the pages
 * measure against.  Assign materialises the full fp32 distance matrix
 * dist[b,i,k] = ||x||^2 + ||c||^2 - 2 x.c in `dist` (device, B*N*K floats,
 * caller-allocated) and then argmins it; update scatters every point into
 * its centroid with one atomicAdd per element ("Flash-KMeans: Fast and
 * Memory-Efficient Exact K-Means" summary, section "Key claims" and "Method").
 * Same outputs and workspace as fkm_assign / fkm_update.  Async. */
FKM_API fkm_status fkm_baseline_assign(int B, int N, int K, int D, int dtype, const void* x,
                               const float* centers, float* dist, int32_t* ids, void* ws,
                               size_t ws_bytes, void* stream);
FKM_API fkm_status fkm_baseline_update(int B, int N, int K, int D, int dtype, const void* x,
                               const int32_t* ids, const float* prev_centers, float* centers,
                               int32_t* counts, void* ws, size_t ws_bytes, void* stream);

/* Progress output of the Lloyd loops ("Flash-KMeans" GitHub README, section
 * "Usage": the verbose argument of batch_kmeans_Euclid).  With level > 0,
 * fkm_lloyd and fkm_lloyd_metric run their stepped loop (also when tol = 0)
 * and print one line per iteration to stderr: the objective of that
 * iteration's assignment summed over the batches, and the largest per-batch
 * centroid shift.  Results are unchanged; the stepped loop syncs every
 * iteration.  Process-wide; level 0 (the default) turns it off. */
FKM_API fkm_status fkm_set_verbose(int level);

/* Stage timing of fkm_lloyd (tracing).  While enabled, fkm_lloyd records CUDA
 * events on its stream (inside its captured graph too) around each stage of
 * every iteration; fkm_profile_read returns the accumulated milliseconds per
 * stage -- [0] assign, [1] argsort, [2] segment bounds + segment sums (+
 * objective), [3] finalize + per-batch reduce, [4] whole iterations -- and
 * the number of iterations timed, and optionally resets them.  Host pointers.
 * Thread-safe; profiling serialises fkm_lloyd calls. */
FKM_API fkm_status fkm_profile(int enable);
FKM_API fkm_status fkm_profile_read(double* stage_ms /*[5]*/, long long* iterations, int reset);

/* Number of kernels this library has launched in this process (graph replays
 * count the kernels the graph holds). */
FKM_API long long fkm_kernel_launches(void);

/* Size of the static device scratch that fkm_assign_noalloc uses (16 MiB). */
#define FKM_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* fkm_assign for callers that cannot allocate device memory.  The paper has no
 * counterpart: this is an interface for code that must not call cudaMalloc at
 * the point it needs an assignment -- code whose device memory belongs to a
 * framework allocator that must not be bypassed there, services that reserve
 * all device memory up front in fixed pools, or plugins that are handed only
 * their inputs and outputs.  Same result as fkm_assign with inertia = NULL, but the
 * scratch (the mean centroids, the rounded centroid offsets, their norm terms
 * and a status word) lives in a
 * file-scope device array of FKM_NOALLOC_SCRATCH_BYTES that every GPU loading
 * the library keeps until the process exits; no workspace is passed and
 * nothing is allocated.
 *   x        device [B,N,D] bf16 or fp16 (fp32 points are rejected: their
 *            split operands need scratch proportional to N)
 *   centers  device [B,K,D] float32;  ids device [B,N] int32 (out)
 * Limit: 256 + B*(4*D + Kp*(2*D + 32)) bytes (each of the three parts
 * rounded up to 256-byte blocks) must fit in FKM_NOALLOC_SCRATCH_BYTES, Kp = K
 * rounded up to 256; larger shapes return FKM_ERR_UNSUPPORTED.  The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress) and
 * raises the kernel's shared-memory limit; make that first call before any
 * stream capture.  The address is kept for the life of the process: a device
 * reset while the library is loaded is not supported.  All calls share the one
 * array, which keeps the last call's contents (the status word is cleared at
 * the start of each call, the rest is rewritten): calls that can overlap on the
 * GPU (other streams, other threads) race with each other, so serialise them.
 * Device-side status (a bounded wait that ran out) is read with
 * fkm_assign_noalloc_status.  Async. */
FKM_API fkm_status fkm_assign_noalloc(int B, int N, int K, int D, int dtype, const void* x,
                                      const float* centers, int32_t* ids, void* stream);

/* Status of the fkm_assign_noalloc calls on the current device (no
 * counterpart in the paper): waits for `stream`, then reads and clears the
 * status word in the static scratch array.  FKM_OK, or FKM_ERR_TIMEOUT when a
 * device-side bounded wait ran out (the ids of that call are then not valid).
 * Allocates nothing; call it on the stream of the fkm_assign_noalloc calls it
 * reports on. */
FKM_API fkm_status fkm_assign_noalloc_status(void* stream);

/* Instrumentation of the Sort-Inverse Update's atomics ("Flash-KMeans：快速且
 * 内存高效精确K-Means聚类" summary, sections 前置知识 / argsort与分段规约 and
 * 方法步骤详情 step (2): one atomic add per segment boundary, O((K + N/B_N) d)
 * in all instead of O(N d)).  Reads the number of fp64 element atomics the
 * segment sums of fkm_update / fkm_lloyd added into the workspace's cluster
 * sums since the count was last reset (a zeroed workspace, the start of each
 * fkm_lloyd call, or a call here with reset != 0), after waiting for `stream`.
 * range_rows (optional) receives B_N, the sorted rows per segment-sum range
 * that an update of n_rows = B*N points uses on the current device: runs that
 * lie inside one range make no atomics, a run that crosses a range boundary
 * makes D per range it touches.  ws: the workspace of those calls (its first
 * 256 bytes hold the count).  Either output may be NULL. */
FKM_API fkm_status fkm_segsum_stats(void* ws, size_t ws_bytes, int64_t n_rows, int reset,
                                    unsigned long long* atomics, int* range_rows,
                                    void* stream);

/* Waits for `stream`, then reads and clears the workspace's status word:
 * FKM_OK, FKM_ERR_TIMEOUT, FKM_ERR_BAD_ID or FKM_ERR_INTERNAL. */
FKM_API fkm_status fkm_sync_status(void* ws, size_t ws_bytes, void* stream);

/* Self-test of failure detection (no counterpart in the pages): launches one
 * kernel whose bounded mbarrier wait is made to run out -- it waits
 * timeout_ns (1 us .. 1 s) for an arrival nobody makes, then sets the
 * timeout bit in the workspace's status word and returns, as every bounded
 * wait in the library does.  A following fkm_sync_status on the same
 * workspace returns FKM_ERR_TIMEOUT, and the context stays usable.  ws:
 * device, >= 256 bytes, 16-byte aligned (its first word is the status).
 * Async. */
FKM_API fkm_status fkm_selftest_wait_timeout(uint64_t timeout_ns, void* ws, size_t ws_bytes,
                                             void* stream);

FKM_API const char* fkm_status_string(fkm_status s);
/* Thread-local text about the last failure in this thread ("" if none). */
FKM_API const char* fkm_last_error(void);
/* Library version string. */
FKM_API const char* fkm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FKM_H_ */
