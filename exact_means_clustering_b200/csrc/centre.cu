// Centring of the points ("Flash-KMeans" GitHub README, section "Centre your
// data"): k-means is translation invariant, so points with a large common
// offset can be clustered after subtracting their per-batch mean, and the
// centroids shifted back.  The README leaves this out of its backend because
// it costs one extra pass over x; here it is a separate, optional call.
//
//   mean       mu[b, d] = fp32((sum over i of x[b, i, d]) / N), the sum in fp64:
//              one block per (batch, run of CENTRE_ROWS rows) sums its rows in
//              order into a partial, and the partials are added in order.
//   subtract   x_out[b, i, d] = RNE_dtype(fp32(x) - mu[b, d]), one fp32
//              subtraction per element, 16 bytes per thread; x_out may be x.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fkm_internal.cuh"

namespace fkm {
namespace {

constexpr int CENTRE_ROWS = 1024;     // rows per partial sum
constexpr int CENTRE_THREADS = 256;

__device__ __forceinline__ float load_f(const void* x, int dtype, int64_t i) {
  if (dtype == FKM_F32) return static_cast<const float*>(x)[i];
  if (dtype == FKM_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(x)[i]);
  return __half2float(static_cast<const __half*>(x)[i]);
}

// grid (partials, B): thread t sums columns t, t + 256, ... of its rows
__global__ void __launch_bounds__(CENTRE_THREADS) centre_partial_kernel(
    const void* __restrict__ x, int dtype, int N, int D, int P, double* __restrict__ part) {
  const int p = blockIdx.x, b = blockIdx.y;
  const int64_t r0 = (int64_t)p * CENTRE_ROWS;
  const int rows = (int)((N - r0) < CENTRE_ROWS ? (N - r0) : CENTRE_ROWS);
  for (int d = threadIdx.x; d < D; d += CENTRE_THREADS) {
    double s = 0.0;
    const int64_t base = ((int64_t)b * N + r0) * D + d;
    for (int i = 0; i < rows; ++i) s += (double)load_f(x, dtype, base + (int64_t)i * D);
    part[((int64_t)b * P + p) * D + d] = s;
  }
}

__global__ void __launch_bounds__(CENTRE_THREADS) centre_mean_kernel(const double* __restrict__ part,
                                                                    int N, int D, int P,
                                                                    float* __restrict__ mu) {
  const int b = blockIdx.x;
  for (int d = threadIdx.x; d < D; d += CENTRE_THREADS) {
    double s = 0.0;
    for (int p = 0; p < P; ++p) s += part[((int64_t)b * P + p) * D + d];
    mu[(int64_t)b * D + d] = (float)(s / (double)N);
  }
}

// one 16-byte vector per thread (D * elem_bytes is a multiple of 16)
template <int DT>
__global__ void __launch_bounds__(CENTRE_THREADS) centre_subtract_kernel(
    const void* x, void* x_out, const float* __restrict__ mu, int N, int D, int64_t nvec) {
  const int64_t v = (int64_t)blockIdx.x * CENTRE_THREADS + threadIdx.x;
  if (v >= nvec) return;
  constexpr int E = DT == FKM_F32 ? 4 : 8;
  const int64_t e0 = v * E;                 // first element
  const int64_t row = e0 / D;
  const int d0 = (int)(e0 - row * D);
  const float* m = mu + (row / N) * D + d0;
  const uint4 in = reinterpret_cast<const uint4*>(x)[v];
  uint4 out;
  if (DT == FKM_F32) {
    out.x = __float_as_uint(__uint_as_float(in.x) - m[0]);
    out.y = __float_as_uint(__uint_as_float(in.y) - m[1]);
    out.z = __float_as_uint(__uint_as_float(in.z) - m[2]);
    out.w = __float_as_uint(__uint_as_float(in.w) - m[3]);
  } else {
    const uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float a, c;
      if (DT == FKM_BF16) {
        a = __uint_as_float(w[k] << 16);
        c = __uint_as_float(w[k] & 0xFFFF0000u);
        const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(a - m[2 * k]));
        const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(c - m[2 * k + 1]));
        o[k] = lo | (hi << 16);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
        const uint32_t lo = __half_as_ushort(__float2half_rn(f.x - m[2 * k]));
        const uint32_t hi = __half_as_ushort(__float2half_rn(f.y - m[2 * k + 1]));
        o[k] = lo | (hi << 16);
      }
    }
    out = make_uint4(o[0], o[1], o[2], o[3]);
  }
  reinterpret_cast<uint4*>(x_out)[v] = out;
}

int64_t centre_partials(int N) { return ceil_div(N, CENTRE_ROWS); }

// out[b, k, d] = fp32(c[b, k, d] + sign * mu[b, d]): one IEEE fp32 addition
// (or subtraction) per element; out may be c.
__global__ void __launch_bounds__(CENTRE_THREADS) shift_centroids_kernel(
    const float* c, const float* __restrict__ mu, float sign, int K, int D, int64_t n,
    float* out) {
  const int64_t e = (int64_t)blockIdx.x * CENTRE_THREADS + threadIdx.x;
  if (e >= n) return;
  const int64_t d = e % D, b = e / ((int64_t)K * D);
  const float m = mu[b * D + d];
  out[e] = sign > 0.0f ? c[e] + m : c[e] - m;
}

}  // namespace
}  // namespace fkm

using namespace fkm;

extern "C" fkm_status fkm_centre_workspace_size(int B, int N, int D, size_t* bytes) {
  if (!bytes || B < 1 || N < 1 || D < 1) {
    set_error("B, N, D must be >= 1 and bytes non-null");
    return FKM_ERR_INVALID_ARG;
  }
  *bytes = (size_t)B * (size_t)centre_partials(N) * (size_t)D * sizeof(double);
  return FKM_OK;
}

extern "C" fkm_status fkm_centre(int B, int N, int D, int dtype, const void* x, float* mu,
                                 void* x_out, void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  FKM_TRY(fkm_centre_workspace_size(B, N, D, &need));
  if (dtype != FKM_F32 && dtype != FKM_F16 && dtype != FKM_BF16) {
    set_error("unknown dtype %d", dtype);
    return FKM_ERR_INVALID_ARG;
  }
  if (((int64_t)D * elem_bytes(dtype)) % 16 != 0 || (int64_t)B * N >= (int64_t(1) << 31) ||
      B > 65535) {   // the partial sums run one grid row per batch
    set_error("D * element size must be a multiple of 16 bytes, B * N < 2^31 and B <= 65535");
    return FKM_ERR_UNSUPPORTED;
  }
  const void* ptrs[] = {x, mu, x_out, ws};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15)) {
      set_error("x, mu, x_out and ws must be non-null and 16-byte aligned");
      return FKM_ERR_INVALID_ARG;
    }
  if (ws_bytes < need) {
    set_error("workspace of %zu bytes is smaller than the %zu required", ws_bytes, need);
    return FKM_ERR_WORKSPACE_TOO_SMALL;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int P = (int)centre_partials(N);
  double* part = static_cast<double*>(ws);
  centre_partial_kernel<<<dim3((unsigned)P, (unsigned)B), CENTRE_THREADS, 0, st>>>(x, dtype, N, D,
                                                                                    P, part);
  centre_mean_kernel<<<(unsigned)B, CENTRE_THREADS, 0, st>>>(part, N, D, P, mu);
  const int64_t nvec = (int64_t)B * N * D * elem_bytes(dtype) / 16;
  const unsigned grid = (unsigned)ceil_div(nvec, CENTRE_THREADS);
  if (dtype == FKM_BF16)
    centre_subtract_kernel<FKM_BF16><<<grid, CENTRE_THREADS, 0, st>>>(x, x_out, mu, N, D, nvec);
  else if (dtype == FKM_F16)
    centre_subtract_kernel<FKM_F16><<<grid, CENTRE_THREADS, 0, st>>>(x, x_out, mu, N, D, nvec);
  else
    centre_subtract_kernel<FKM_F32><<<grid, CENTRE_THREADS, 0, st>>>(x, x_out, mu, N, D, nvec);
  note_launch(3);
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

extern "C" fkm_status fkm_shift_centroids(int B, int K, int D, const float* centers,
                                          const float* mu, int sign, float* out, void* stream) {
  if (B < 1 || K < 1 || D < 1 || (sign != 1 && sign != -1)) {
    set_error("B, K, D must be >= 1 and sign +1 or -1");
    return FKM_ERR_INVALID_ARG;
  }
  if (!centers || !mu || !out) {
    set_error("centers, mu and out must be non-null");
    return FKM_ERR_INVALID_ARG;
  }
  const int64_t n = (int64_t)B * K * D;
  shift_centroids_kernel<<<(unsigned)ceil_div(n, CENTRE_THREADS), CENTRE_THREADS, 0,
                           static_cast<cudaStream_t>(stream)>>>(centers, mu, (float)sign, K, D,
                                                                n, out);
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}
