// The comparison point the pages measure against -- NOT the method.
//
// "Flash-KMeans: Fast and Memory-Efficient Exact K-Means" summary, sections
// "Key claims" and "Method": a standard iteration writes the full N x K
// distance matrix to HBM and reads it back for the argmin, then updates the
// centroids with scatter-style atomic adds keyed by cluster id (the same
// page quotes ~50 GB/s effective bandwidth for that update on H200).
//
//   fkm_baseline_assign  tensor-core distances written to dist[B, N, K]
//                        (the assign kernel's materialising mode), then a
//                        one-warp-per-row argmin that reads them back.
//   fkm_baseline_update  one fp32 atomicAdd per point per element into the
//                        cluster sums plus one count atomic per point, then a
//                        divide (empty clusters keep the previous centroid).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fkm_internal.cuh"

namespace fkm {
namespace {

__global__ void argmin_rows_kernel(const float* __restrict__ dist, int64_t rows, int K,
                                   int32_t* __restrict__ ids) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* d = dist + row * K;
  float best = INFINITY;
  int bi = K;
  for (int k = lane; k < K; k += 32) {
    const float v = d[k];
    if (v < best) { best = v; bi = k; }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov < best || (ov == best && oi < bi)) { best = ov; bi = oi; }
  }
  if (lane == 0) ids[row] = bi < K ? bi : 0;
}

__device__ __forceinline__ float load_elem(const void* x, int dtype, int64_t i) {
  if (dtype == FKM_F32) return static_cast<const float*>(x)[i];
  if (dtype == FKM_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(x)[i]);
  return __half2float(static_cast<const __half*>(x)[i]);
}

// one thread per (point, element)
__global__ void scatter_kernel(const void* __restrict__ x, int dtype, const int32_t* __restrict__ ids,
                               int64_t BN, int N, int K, int D, float* sums, int32_t* cnt,
                               int* status) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= BN * D) return;
  const int64_t row = e / D;
  const int d = (int)(e % D);
  const int id = ids[row];
  if (id < 0 || id >= K) {
    if (d == 0) atomicOr(status, ST_BAD_ID);
    return;
  }
  const int64_t key = (row / N) * K + id;
  atomicAdd(&sums[key * D + d], load_elem(x, dtype, e));
  if (d == 0) atomicAdd(&cnt[key], 1);
}

__global__ void divide_kernel(const float* __restrict__ sums, const int32_t* __restrict__ cnt,
                              const float* __restrict__ prev, float* __restrict__ centers,
                              int32_t* __restrict__ counts, int64_t BK, int D) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= BK * D) return;
  const int64_t key = e / D;
  const int n = cnt[key];
  centers[e] = n > 0 ? sums[e] / (float)n : prev[e];
  if (e % D == 0) counts[key] = n;
}

}  // namespace

fkm_status launch_baseline_argmin(const float* dist, int64_t rows, int K, int32_t* ids,
                                  cudaStream_t st) {
  const int wpb = 8;
  argmin_rows_kernel<<<(unsigned)ceil_div(rows, wpb), wpb * 32, 0, st>>>(dist, rows, K, ids);
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

fkm_status launch_baseline_update(const void* x, int dtype, const int32_t* ids, int B, int N,
                                  int K, int D, float* sums, int32_t* cnt, const float* prev,
                                  float* centers, int32_t* counts, int* status, cudaStream_t st) {
  const int64_t BK = (int64_t)B * K, BN_ = (int64_t)B * N;
  FKM_CUDA_TRY(cudaMemsetAsync(sums, 0, sizeof(float) * BK * D, st));
  FKM_CUDA_TRY(cudaMemsetAsync(cnt, 0, sizeof(int32_t) * BK, st));
  scatter_kernel<<<(unsigned)ceil_div(BN_ * D, 256), 256, 0, st>>>(x, dtype, ids, BN_, N, K, D,
                                                                   sums, cnt, status);
  divide_kernel<<<(unsigned)ceil_div(BK * D, 256), 256, 0, st>>>(sums, cnt, prev, centers, counts,
                                                                 BK, D);
  note_launch(2);
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

}  // namespace fkm
