// Out-of-core Lloyd: points stay in host pinned memory and stream through the
// device in chunks ("Flash-KMeans" GitHub README, section "Large tensor
// Benchmark": data in CPU pinned memory, transferred chunk by chunk;
// "Flash-KMeans：快速且内存高效精确K-Means聚类" summary, section 方法步骤详情
// step (3): CUDA streams, double buffering, the next chunk transferred while
// the current one is processed).
//
// Two device chunk buffers; a copy stream issues cudaMemcpyAsync (host pinned
// -> device) into one while the caller's stream runs, on the other, the
// assign kernel and a chunk-local sort-inverse update whose segment sums all
// go to fp64 accumulators (a run of one chunk is never a whole cluster).
// After the last chunk one finalize divides, keeps empty clusters, computes
// the shift and re-quantises the centroids.  Events order the two streams;
// the copy of the next iteration's first chunk waits only for its buffer, so
// it overlaps the previous iteration's finalize (the README's prefetch of the
// first block of the next iteration, "Multi-GPU Support").
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "fkm_internal.cuh"

namespace fkm {

namespace {

template <typename T>
__global__ void accumulate_counts_kernel(const int32_t* __restrict__ segstart,
                                         const int32_t* __restrict__ segend, int K,
                                         T* __restrict__ acc) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < K) acc[k] += (T)(segend[k] - segstart[k]);
}

struct HostLayout {
  int B, N, K, D, dtype, Kp, Dp, Dq;
  bool split;
  int64_t R;              // chunk rows (multiple of BM)
  int chunks_per_batch;
  int tiles_per_chunk;
  int key_bits;
  size_t status, xbuf[2], mvec, cq, caug, xs, xn, keys0, vals0, keys1, vals1, hist, hist_part,
      segstart, segend, sums64, counts_acc, shiftk, cnorm, objk, cbuf, total;
};

int bits_for_value(int64_t v) {
  int b = 0;
  while ((int64_t(1) << b) <= v) ++b;
  return b < 1 ? 1 : b;
}

fkm_status make_host_layout(int B, int N, int K, int D, int dtype, int64_t chunk_rows,
                            HostLayout* out) {
  size_t probe = 0;
  FKM_TRY(fkm_workspace_size(B, 1, K, D, dtype, &probe));  // shape validation
  if ((int64_t)B * N >= (int64_t(1) << 31)) {
    set_error("B*N must stay below 2^31");
    return FKM_ERR_UNSUPPORTED;
  }
  if (N < 1 || chunk_rows < 1) {
    set_error("N and chunk_rows must be >= 1");
    return FKM_ERR_INVALID_ARG;
  }
  HostLayout l;
  l.B = B;
  l.N = N;
  l.K = K;
  l.D = D;
  l.dtype = dtype;
  l.split = dtype == FKM_F32;
  l.Kp = (int)round_up(K, BN);
  l.Dp = (int)round_up(D, 8);
  l.Dq = l.split ? 2 * l.Dp : D;
  int64_t R = round_up(chunk_rows, BM);
  if (R > round_up(N, BM)) R = round_up(N, BM);
  l.R = R;
  l.chunks_per_batch = (int)ceil_div(N, R);
  l.tiles_per_chunk = (int)(R / BM);
  l.key_bits = bits_for_value(K);
  const size_t s = (size_t)elem_bytes(dtype);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t BK = (size_t)B * K;
  l.status = take(256);
  l.xbuf[0] = take((size_t)R * D * s);
  l.xbuf[1] = take((size_t)R * D * s);
  l.mvec = take((size_t)B * D * 4);
  l.cq = take((size_t)B * l.Kp * l.Dq * 2);
  l.caug = take((size_t)B * l.Kp * AUG_SLAB * 2);
  l.xs = take(l.split ? (size_t)R * l.Dq * 2 : 0);
  l.xn = take((size_t)R * 4);
  l.keys0 = take((size_t)R * 4);
  l.vals0 = take((size_t)R * 4);
  l.keys1 = take((size_t)R * 4);
  l.vals1 = take((size_t)R * 4);
  l.hist = take((size_t)ceil_div(R, SORT_TILE) * RADIX_BINS * 4);
  l.hist_part = take(argsort_scratch_words(R) * 4);
  l.segstart = take((size_t)K * 4);
  l.segend = take((size_t)K * 4);
  l.sums64 = take(BK * D * 8);
  l.counts_acc = take(BK * 4);
  l.shiftk = take(BK * 8);
  l.cnorm = take(BK * 8);   // cosine: centroid row norms
  l.objk = take(BK * 8);    // dot / cosine: each cluster's share of the objective
  l.cbuf = take(2 * BK * D * 4);
  l.total = off;
  *out = l;
  return FKM_OK;
}

struct StreamSet {
  cudaStream_t copy = nullptr;
  cudaEvent_t copied[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr}, start = nullptr;
  ~StreamSet() {
    for (int i = 0; i < 2; ++i) {
      if (copied[i]) cudaEventDestroy(copied[i]);
      if (freed[i]) cudaEventDestroy(freed[i]);
    }
    if (start) cudaEventDestroy(start);
    if (copy) cudaStreamDestroy(copy);
  }
};

// Host-side fault injection for the failure-detection tests (off unless the
// environment asks for it): FKM_FAULT_INJECT=h2d@chunk:<n> makes the copy of
// the n-th streamed chunk (counted over the whole call) fail as a CUDA error
// would, before it is issued.  Nothing is done on the GPU to cause it.
int64_t injected_h2d_fault_chunk() {
  const char* v = std::getenv("FKM_FAULT_INJECT");
  long long n = -1;
  if (v && std::sscanf(v, "h2d@chunk:%lld", &n) == 1 && n >= 0) return (int64_t)n;
  return -1;
}

// Partial mode (one shard of a data-parallel run): one pass over the chunks
// with the given centroids, adding the per-cluster sums, counts and objective
// to the caller's buffers instead of finalizing.
struct HostPartial {
  double* sums;
  double* counts;
  double* obj;
  int flags;   // FKM_HOST_COPY_AT_ONCE
};

}  // namespace
}  // namespace fkm

using namespace fkm;

static fkm_status lloyd_host_impl(int B, int N, int K, int D, int dtype, int metric,
                                  const void* x_host, const float* init_centers, int max_iters,
                                  float tol, int64_t chunk_rows, int32_t* ids, float* centers,
                                  int32_t* counts, double* inertia, int* n_iter, void* ws,
                                  size_t ws_bytes, void* stream, const HostPartial* part);

extern "C" {

fkm_status fkm_host_workspace_size(int B, int N, int K, int D, int dtype, int64_t chunk_rows,
                                   size_t* bytes) {
  if (!bytes) {
    set_error("bytes is null");
    return FKM_ERR_INVALID_ARG;
  }
  HostLayout L;
  FKM_TRY(make_host_layout(B, N, K, D, dtype, chunk_rows, &L));
  *bytes = L.total;
  return FKM_OK;
}

fkm_status fkm_lloyd_host(int B, int N, int K, int D, int dtype, const void* x_host,
                          const float* init_centers, int max_iters, float tol,
                          int64_t chunk_rows, int32_t* ids, float* centers, int32_t* counts,
                          double* inertia, int* n_iter, void* ws, size_t ws_bytes, void* stream) {
  return lloyd_host_impl(B, N, K, D, dtype, FKM_METRIC_EUCLID, x_host, init_centers, max_iters,
                         tol, chunk_rows, ids, centers, counts, inertia, n_iter, ws, ws_bytes,
                         stream, nullptr);
}

fkm_status fkm_lloyd_host_metric(int B, int N, int K, int D, int dtype, int metric,
                                 const void* x_host, const float* init_centers, int max_iters,
                                 float tol, int64_t chunk_rows, int32_t* ids, float* centers,
                                 int32_t* counts, double* objective, int* n_iter, void* ws,
                                 size_t ws_bytes, void* stream) {
  if (metric != FKM_METRIC_EUCLID && metric != FKM_METRIC_DOT && metric != FKM_METRIC_COSINE) {
    set_error("unknown metric %d", metric);
    return FKM_ERR_INVALID_ARG;
  }
  return lloyd_host_impl(B, N, K, D, dtype, metric, x_host, init_centers, max_iters, tol,
                         chunk_rows, ids, centers, counts, objective, n_iter, ws, ws_bytes,
                         stream, nullptr);
}

fkm_status fkm_partial_update_host(int B, int N, int K, int D, int dtype, const void* x_host,
                                   const float* centers, int64_t chunk_rows, int32_t* ids,
                                   double* sums, double* counts, double* obj, int flags,
                                   void* ws, size_t ws_bytes, void* stream) {
  if (flags & ~FKM_HOST_COPY_AT_ONCE) {
    set_error("unknown flags 0x%x", flags);
    return FKM_ERR_INVALID_ARG;
  }
  if (!sums || !counts || (reinterpret_cast<uintptr_t>(sums) & 15) ||
      (reinterpret_cast<uintptr_t>(counts) & 15) ||
      (obj && (reinterpret_cast<uintptr_t>(obj) & 15))) {
    set_error("sums and counts must be non-null; sums, counts and obj 16-byte aligned");
    return FKM_ERR_INVALID_ARG;
  }
  HostPartial part{sums, counts, obj, flags};
  int n_iter = 0;
  // counts is only checked for null and alignment on this path: the partial
  // pass adds into part.counts (fp64), never into the int32 output
  return lloyd_host_impl(B, N, K, D, dtype, FKM_METRIC_EUCLID, x_host, centers, 1, 0.0f,
                         chunk_rows, ids, const_cast<float*>(centers),
                         reinterpret_cast<int32_t*>(counts), obj, &n_iter, ws, ws_bytes, stream,
                         &part);
}

}  // extern "C"

// metric: FKM_METRIC_EUCLID, or dot / cosine k-means (fkm_lloyd_metric's
// arithmetic: operands of the scaled rows, no bias, every cluster's objective
// share from its sums in the finalize; inertia then receives that objective).
static fkm_status lloyd_host_impl(int B, int N, int K, int D, int dtype, int metric,
                                  const void* x_host, const float* init_centers, int max_iters,
                                  float tol, int64_t chunk_rows, int32_t* ids, float* centers,
                                  int32_t* counts, double* inertia, int* n_iter, void* ws,
                                  size_t ws_bytes, void* stream, const HostPartial* part) {
  HostLayout L;
  FKM_TRY(make_host_layout(B, N, K, D, dtype, chunk_rows, &L));
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15) || ws_bytes < L.total) {
    set_error("workspace null, misaligned or smaller than the %zu bytes required", L.total);
    return (ws && ws_bytes < L.total) ? FKM_ERR_WORKSPACE_TOO_SMALL : FKM_ERR_INVALID_ARG;
  }
  const void* ptrs[] = {x_host, init_centers, ids, centers, counts};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15)) {
      set_error("a required pointer is null or not 16-byte aligned");
      return FKM_ERR_INVALID_ARG;
    }
  if (inertia && (reinterpret_cast<uintptr_t>(inertia) & 15)) {
    set_error("inertia is not 16-byte aligned");
    return FKM_ERR_INVALID_ARG;
  }
  if (!n_iter || max_iters < 1 || !(tol >= 0.0f)) {
    set_error("n_iter must be non-null, max_iters >= 1 and tol >= 0");
    return FKM_ERR_INVALID_ARG;
  }
  cudaPointerAttributes pa;
  if (cudaPointerGetAttributes(&pa, x_host) != cudaSuccess || pa.type != cudaMemoryTypeHost) {
    cudaGetLastError();
    set_error("x_host must be page-locked host memory (cudaHostAlloc / cudaHostRegister)");
    return FKM_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  auto at = [&](size_t off) { return static_cast<void*>(w + off); };
  int* status = static_cast<int*>(at(L.status));
  double* max_shift = reinterpret_cast<double*>(w + L.status + 64);
  const size_t s = (size_t)elem_bytes(dtype);
  const size_t cbytes = (size_t)B * K * D * sizeof(float);
  float* cA = static_cast<float*>(at(L.cbuf));
  float* cB = cA + (size_t)B * K * D;
  double* sums64 = part ? part->sums : static_cast<double*>(at(L.sums64));
  int32_t* counts_acc = static_cast<int32_t*>(at(L.counts_acc));

  StreamSet ss;
  FKM_CUDA_TRY(cudaStreamCreateWithFlags(&ss.copy, cudaStreamNonBlocking));
  for (int i = 0; i < 2; ++i) {
    FKM_CUDA_TRY(cudaEventCreateWithFlags(&ss.copied[i], cudaEventDisableTiming));
    FKM_CUDA_TRY(cudaEventCreateWithFlags(&ss.freed[i], cudaEventDisableTiming));
  }
  FKM_CUDA_TRY(cudaEventCreateWithFlags(&ss.start, cudaEventDisableTiming));
  FKM_TRY(assign_prepare());

  FKM_CUDA_TRY(cudaMemsetAsync(status, 0, 256, st));
  if (!part) FKM_CUDA_TRY(cudaMemsetAsync(sums64, 0, (size_t)B * K * D * 8, st));
  FKM_CUDA_TRY(cudaMemcpyAsync(cA, init_centers, cbytes, cudaMemcpyDeviceToDevice, st));
  float* mvec = static_cast<float*>(at(L.mvec));
  const bool euclid = metric == FKM_METRIC_EUCLID;
  double* cnorm = static_cast<double*>(at(L.cnorm));
  double* objk = static_cast<double*>(at(L.objk));
  FKM_TRY(launch_prep_centroids(cA, B, K, L.Kp, D, dtype, mvec, at(L.cq),
                                at(L.caug), st, metric, cnorm));
  // The copy stream may only touch the workspace after the caller's earlier
  // work, unless the caller vouches that the chunk buffers are idle: then
  // the first chunk's copy starts at once and overlaps whatever is still
  // queued on the caller's stream (in a data-parallel loop, the previous
  // iteration's all-reduce and finalize).
  if (!(part && (part->flags & FKM_HOST_COPY_AT_ONCE))) {
    FKM_CUDA_TRY(cudaEventRecord(ss.start, st));
    FKM_CUDA_TRY(cudaStreamWaitEvent(ss.copy, ss.start, 0));
  }

  int done = 0;
  int64_t chunk_no = 0;
  const int64_t fault_chunk = injected_h2d_fault_chunk();
  for (int t = 0; t < max_iters; ++t) {
    float* cur = (t & 1) ? cB : cA;
    float* nxt = (t & 1) ? cA : cB;
    if (!part) {   // a partial pass adds to the caller's buffers
      FKM_CUDA_TRY(cudaMemsetAsync(counts_acc, 0, (size_t)B * K * 4, st));
      if (inertia) FKM_CUDA_TRY(cudaMemsetAsync(inertia, 0, (size_t)B * 8, st));
    }
    for (int b = 0; b < B; ++b) {
      for (int c = 0; c < L.chunks_per_batch; ++c, ++chunk_no) {
        const int buf = (int)(chunk_no & 1);
        const int64_t n0 = (int64_t)c * L.R;
        const int rows = (int)((N - n0) < L.R ? (N - n0) : L.R);
        void* xb = at(L.xbuf[buf]);
        FKM_CUDA_TRY(cudaStreamWaitEvent(ss.copy, ss.freed[buf], 0));
        if (chunk_no == fault_chunk) {
          set_error("injected fault (FKM_FAULT_INJECT): host-to-device copy of chunk %lld",
                    (long long)chunk_no);
          return FKM_ERR_CUDA;
        }
        FKM_CUDA_TRY(cudaMemcpyAsync(xb,
                                     static_cast<const char*>(x_host) +
                                         ((size_t)b * N + n0) * D * s,
                                     (size_t)rows * D * s, cudaMemcpyHostToDevice, ss.copy));
        FKM_CUDA_TRY(cudaEventRecord(ss.copied[buf], ss.copy));
        FKM_CUDA_TRY(cudaStreamWaitEvent(st, ss.copied[buf], 0));

        if (L.split) FKM_TRY(launch_points_prep(xb, rows, D, dtype, at(L.xs), nullptr, st));
        int32_t* ids_c = ids + (size_t)b * N + n0;
        AssignArgs a;
        a.B = 1;
        a.N = rows;
        a.K = K;
        a.Kp = L.Kp;
        a.D = D;
        a.dtype = dtype;
        a.split = L.split;
        a.xq = L.split ? at(L.xs) : xb;
        a.x_row_elems = L.split ? L.Dq : D;
        a.cq = static_cast<const char*>(at(L.cq)) + (size_t)b * L.Kp * L.Dq * 2;
        a.caug = static_cast<const char*>(at(L.caug)) + (size_t)b * L.Kp * AUG_SLAB * 2;
        a.xn = nullptr;
        a.ids = ids_c;
        a.status = status;
        FKM_TRY(launch_assign(a, st));

        SortArgs so;
        so.ids = ids_c;
        so.N = rows;
        so.K = K;
        so.n = rows;
        so.key_bits = L.key_bits;
        so.keys0 = static_cast<int32_t*>(at(L.keys0));
        so.vals0 = static_cast<int32_t*>(at(L.vals0));
        so.keys1 = static_cast<int32_t*>(at(L.keys1));
        so.vals1 = static_cast<int32_t*>(at(L.vals1));
        so.hist = static_cast<uint32_t*>(at(L.hist));
        so.hist_part = static_cast<uint32_t*>(at(L.hist_part));
        so.status = status;
        FKM_TRY(launch_argsort_ids(so, st));
        int32_t* segstart = static_cast<int32_t*>(at(L.segstart));
        int32_t* segend = static_cast<int32_t*>(at(L.segend));
        FKM_TRY(clear_seg_bounds(K, segstart, segend, st));   // the segment sums write them
        ObjArgs oa;
        oa.K = K;
        // the similarity objectives come from the cluster sums in the finalize
        oa.obj = (inertia && euclid) ? inertia + b : nullptr;
        if (L.split) {
          oa.chat = cur + (size_t)b * K * D;
          oa.chat_bstride = 0;
        } else {
          oa.chat = static_cast<const char*>(at(L.cq)) + (size_t)b * L.Kp * D * 2;
          oa.chat_bstride = 0;
          oa.m = mvec + (size_t)b * D;
        }
        FKM_TRY(launch_segsum(xb, dtype, D, so.keys_out, so.vals_out, rows, K,
                              sums64 + (size_t)b * K * D, nullptr, true, oa, st, 0, nullptr,
                              segstart, segend, status));
        if (part)
          accumulate_counts_kernel<double><<<(unsigned)ceil_div(K, 256), 256, 0, st>>>(
              segstart, segend, K, part->counts + (size_t)b * K);
        else
          accumulate_counts_kernel<int32_t><<<(unsigned)ceil_div(K, 256), 256, 0, st>>>(
              segstart, segend, K, counts_acc + (size_t)b * K);
        note_launch();
        FKM_CUDA_TRY(cudaGetLastError());
        FKM_CUDA_TRY(cudaEventRecord(ss.freed[buf], st));
      }
    }
    if (part) {
      done = 1;
      break;
    }
    if (euclid) {
      FKM_TRY(launch_finalize(B, K, D, nullptr, nullptr, counts_acc, sums64, cur, nxt, counts,
                              static_cast<double*>(at(L.shiftk)), st));
    } else {
      FKM_TRY(launch_finalize_sim(B, K, D, metric, nullptr, nullptr, sums64, cur, nxt, counts,
                                  static_cast<double*>(at(L.shiftk)), objk, st, SEG_RANGE,
                                  counts_acc));
      if (inertia) FKM_TRY(launch_batch_reduce(B, K, objk, inertia, nullptr, st));
    }
    FKM_TRY(launch_prep_centroids(nxt, B, K, L.Kp, D, dtype, mvec, at(L.cq),
                                  at(L.caug), st, metric, cnorm));
    if (tol > 0.0f) FKM_CUDA_TRY(cudaMemsetAsync(max_shift, 0, sizeof(double), st));
    FKM_TRY(launch_batch_reduce(B, K, static_cast<double*>(at(L.shiftk)), nullptr,
                                tol > 0.0f ? max_shift : nullptr, st));
    done = t + 1;
    if (tol > 0.0f) {
      double mx = 0.0;
      FKM_CUDA_TRY(cudaMemcpyAsync(&mx, max_shift, sizeof(double), cudaMemcpyDeviceToHost, st));
      FKM_CUDA_TRY(cudaStreamSynchronize(st));
      if (mx < (double)tol) break;
    }
  }
  float* last = (done & 1) ? cB : cA;
  if (!part) FKM_CUDA_TRY(cudaMemcpyAsync(centers, last, cbytes, cudaMemcpyDeviceToDevice, st));
  int host_status = 0;
  FKM_CUDA_TRY(cudaMemcpyAsync(&host_status, status, sizeof(int), cudaMemcpyDeviceToHost, st));
  FKM_CUDA_TRY(cudaStreamSynchronize(st));
  FKM_CUDA_TRY(cudaStreamSynchronize(ss.copy));
  *n_iter = done;
  if (host_status & ST_TIMEOUT) {
    set_error("a device-side bounded wait ran out");
    return FKM_ERR_TIMEOUT;
  }
  if (host_status & ST_OOB) {
    set_error("checked build: a kernel met an out-of-range gather or scatter index");
    return FKM_ERR_INTERNAL;
  }
  if (host_status) {
    set_error("device status 0x%x", host_status);
    return FKM_ERR_INTERNAL;
  }
  return FKM_OK;
}
