// Data-parallel Lloyd over several GPUs ("Flash-KMeans" GitHub README,
// section "Multi-GPU Support"): the N points of every problem are split into
// contiguous shards, one per GPU; each GPU assigns its shard and forms the
// shard's per-cluster sums and counts with the sort-inverse update; the sums
// and counts (a few MB) are reduced across the GPUs; and every GPU forms the
// same new centroids from the reduced sums.  These two calls are the
// per-shard halves of that iteration; the reduction between them is the
// caller's: sums, counts and objective are all fp64, so the caller can lay
// them out in one buffer and reduce it with one all-reduce.
#include "fkm_internal.cuh"

namespace fkm {
namespace {

__global__ void add_counts_kernel(const int32_t* __restrict__ segstart,
                                  const int32_t* __restrict__ segend, int64_t keys,
                                  double* __restrict__ counts) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k < keys) counts[k] += (double)(segend[k] - segstart[k]);
}

fkm_status aligned_or_null(const void* p, const char* name) {
  if (p && (reinterpret_cast<uintptr_t>(p) & 15)) {
    set_error("%s is not 16-byte aligned", name);
    return FKM_ERR_INVALID_ARG;
  }
  return FKM_OK;
}

}  // namespace

fkm_status shard_partial_update(const Layout& L, const void* x, const int32_t* ids,
                                const float* prev, double* sums, double* counts, double* obj,
                                void* ws, cudaStream_t st);

}  // namespace fkm

using namespace fkm;

extern "C" fkm_status fkm_partial_update(int B, int N, int K, int D, int dtype, const void* x,
                                         const int32_t* ids, const float* prev, double* sums,
                                         double* counts, double* obj, void* ws, size_t ws_bytes,
                                         void* stream) {
  size_t need = 0;
  FKM_TRY(fkm_workspace_size(B, N, K, D, dtype, &need));
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15)) {
    set_error("workspace null, misaligned or smaller than the %zu bytes required", need);
    return (ws && ws_bytes < need) ? FKM_ERR_WORKSPACE_TOO_SMALL : FKM_ERR_INVALID_ARG;
  }
  if (!x || !ids || !prev || !sums || !counts) {
    set_error("x, ids, prev, sums and counts must be non-null");
    return FKM_ERR_INVALID_ARG;
  }
  const void* ptrs[] = {x, ids, prev, sums, counts, obj};
  const char* names[] = {"x", "ids", "prev", "sums", "counts", "obj"};
  for (int i = 0; i < 6; ++i) FKM_TRY(aligned_or_null(ptrs[i], names[i]));
  Layout L;
  FKM_TRY(make_layout(B, N, K, D, dtype, &L));
  return shard_partial_update(L, x, ids, prev, sums, counts, obj, ws,
                              static_cast<cudaStream_t>(stream));
}

extern "C" fkm_status fkm_finalize_sums(int B, int K, int D, const double* sums,
                                        const double* counts, const float* prev, float* centers,
                                        int32_t* counts_out, double* shift, void* ws,
                                        size_t ws_bytes, void* stream) {
  if (B < 1 || K < 1 || D < 1 || (int64_t)B * K >= (int64_t(1) << 31)) {
    set_error("B, K, D must be >= 1 and B*K < 2^31");
    return FKM_ERR_INVALID_ARG;
  }
  const size_t need = 256 + (size_t)B * K * sizeof(double);
  if (!ws || ws_bytes < need || !sums || !counts || !prev || !centers) {
    set_error("sums, counts, prev, centers and a workspace of >= %zu bytes are required", need);
    return (ws && ws_bytes < need) ? FKM_ERR_WORKSPACE_TOO_SMALL : FKM_ERR_INVALID_ARG;
  }
  if (prev == centers) {
    set_error("centers must not alias prev");
    return FKM_ERR_INVALID_ARG;
  }
  const void* ptrs[] = {sums, counts, prev, centers, shift, ws, counts_out};
  const char* names[] = {"sums", "counts", "prev", "centers", "shift", "ws", "counts_out"};
  for (int i = 0; i < 7; ++i) FKM_TRY(aligned_or_null(ptrs[i], names[i]));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  double* shiftk = reinterpret_cast<double*>(static_cast<char*>(ws) + 256);
  FKM_TRY(launch_finalize(B, K, D, nullptr, nullptr, nullptr, const_cast<double*>(sums), prev,
                          centers, counts_out, shiftk, st, SEG_RANGE, /*clear_sums=*/false,
                          counts));
  if (shift) FKM_TRY(launch_batch_reduce(B, K, shiftk, shift, nullptr, st));
  return FKM_OK;
}

namespace fkm {

fkm_status shard_partial_update(const Layout& L, const void* x, const int32_t* ids,
                                const float* prev, double* sums, double* counts, double* obj,
                                void* wsp, cudaStream_t st) {
  char* w = static_cast<char*>(wsp);
  auto at = [&](size_t off) { return static_cast<void*>(w + off); };
  // the objective measures against c_hat of prev, the assign operand
  if (obj && !L.split)
    FKM_TRY(launch_prep_centroids(prev, L.B, L.K, L.Kp, L.D, L.dtype,
                                  static_cast<float*>(at(L.mvec)), at(L.cq), at(L.caug), st));
  SortArgs s;
  s.ids = ids;
  s.N = L.N;
  s.K = L.K;
  s.n = L.n_sort;
  s.key_bits = L.key_bits;
  s.keys0 = static_cast<int32_t*>(at(L.keys0));
  s.vals0 = static_cast<int32_t*>(at(L.vals0));
  s.keys1 = static_cast<int32_t*>(at(L.keys1));
  s.vals1 = static_cast<int32_t*>(at(L.vals1));
  s.hist = static_cast<uint32_t*>(at(L.hist));
  s.hist_part = static_cast<uint32_t*>(at(L.hist_part));
  s.status = static_cast<int*>(at(L.status));
  const int BK = L.B * L.K;
  int32_t* segstart = static_cast<int32_t*>(at(L.segstart));
  int32_t* segend = static_cast<int32_t*>(at(L.segend));
  if (L.count_sort) {
    FKM_TRY(launch_count_sort_ids(s, L.B, segstart, segend, st));
  } else {   // the segment sums write the bounds
    FKM_TRY(launch_argsort_ids(s, st));
    FKM_TRY(clear_seg_bounds(BK, segstart, segend, st));
  }
  ObjArgs oa;
  oa.K = L.K;
  oa.obj = obj;
  if (L.split) {
    oa.chat = prev;
    oa.chat_bstride = (int64_t)L.K * L.D;
  } else {
    oa.chat = at(L.cq);
    oa.chat_bstride = (int64_t)L.Kp * L.D;
    oa.m = static_cast<float*>(at(L.mvec));
  }
  FKM_TRY(launch_segsum(x, L.dtype, L.D, s.keys_out, s.vals_out, L.n_sort, BK, sums, nullptr,
                        true, oa, st, 0, nullptr, L.count_sort ? nullptr : segstart,
                        L.count_sort ? nullptr : segend, static_cast<int*>(at(L.status))));
  add_counts_kernel<<<(unsigned)ceil_div(BK, 256), 256, 0, st>>>(segstart, segend, BK, counts);
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

}  // namespace fkm
