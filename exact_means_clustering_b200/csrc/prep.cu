// Operand preparation for the assign kernel.
//
//  center: per batch the mean centroid m (fp64 sum over k in a fixed order --
//    32 strided partial sums, then their sum -- divided by K, rounded to fp32).  The assignment works on offsets from m:
//    k-means is translation invariant ("Flash-KMeans" README, section "Centre
//    your data"), and with the offsets small the tensor-core products and
//    their fp32 accumulation keep their precision even for data far from the
//    origin.
//  prep_centroids: delta = fp32(c - m); q(delta) = delta rounded (RNE) to the
//    points' 16-bit type, laid out [B, Kp, D] for TMA; and the norm term
//    n = ||q(delta)||^2 + 2 m.q(delta) (fp64), stored as the bias slab
//    [-n/2 in three 16-bit parts, 0 x 13] that one extra tensor-core product
//    adds to x.q(delta).  Up to terms constant per point, n - 2 x.q(delta) is
//    ||x - c_hat||^2 with c_hat = m + q(delta), so the argmax of
//    x.q(delta) - n/2 is the nearest centroid ("Flash-KMeans：快速且内存高效精确
//    K-Means聚类" summary, section 方法步骤详情 step (1), which precomputes the
//    norms).  Padding rows k >= K are zero (their columns are masked).  For
//    fp32 points delta is split into bf16 hi and lo = bf16(delta - hi), rows
//    [hi | lo], and the norm term uses the fp32 delta.
//  dot-product and cosine k-means (the README lists both beside the
//    Euclidean one): the score is x.c_hat, and x.m is the same for every
//    centroid of a point, so the argmax of x.q(delta) alone picks the most
//    similar centroid -- the bias slab is zero.  For cosine the rows are
//    first scaled to unit length, u = fp32(c / ||c||) with the norm in fp64,
//    and m, delta and q() are formed from u.
//  points_prep: for fp32 points, the bf16 [hi | lo] split rows the tensor
//    cores consume (each half padded to a multiple of 8 elements); optionally
//    ||x - m||^2 per point (fp64 sum rounded to fp32), which only the
//    distance-materialising comparison path needs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fkm_internal.cuh"

namespace fkm {
namespace {

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// A centroid element as the assignment sees it: c itself, or for cosine
// k-means c / ||c|| rounded to fp32 (a zero row stays zero).
__device__ __forceinline__ float metric_elem(float c, const double* cn, int64_t row) {
  if (!cn) return c;
  const double n = cn[row];
  return n > 0.0 ? (float)((double)c / n) : 0.0f;
}

// ||c|| of every centroid row (fp64 sum of squares); one warp per row.
__global__ void row_norms_kernel(const float* __restrict__ c, int64_t rows, int D,
                                 double* __restrict__ cn) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  double s = 0.0;
  for (int d = lane; d < D; d += 32) {
    const double v = (double)c[row * D + d];
    s += v * v;
  }
  s = warp_sum(s);
  if (lane == 0) cn[row] = sqrt(s);
}

// m[b][d] = fp32(S / K) with S summed in fp64 in a fixed order that does not
// depend on the launch: 32 partial sums P_w = sum over k = w, w+32, w+64, ...
// (each in ascending k), then S = P_0 + P_1 + ... + P_31 in that order.
// Block (b, 32-dimension group) of 32 warps: warp w forms P_w for the 32
// dimensions of its lanes (coalesced rows), warp 0 adds the partials.
__global__ void __launch_bounds__(1024) center_kernel(const float* __restrict__ c, int B, int K,
                                                      int D, float* __restrict__ m,
                                                      const double* __restrict__ cn) {
  __shared__ double part[32][33];
  const int b = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int d = blockIdx.y * 32 + lane;
  double s = 0.0;
  if (d < D) {
    const float* p = c + (int64_t)b * K * D + d;
    const int64_t row0 = (int64_t)b * K;
    int k = w;
    // sixteen rows' loads in flight at once, added in the same ascending order
    for (; k + 15 * 32 < K; k += 16 * 32) {
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = p[(int64_t)(k + 32 * j) * D];
#pragma unroll
      for (int j = 0; j < 16; ++j) s += (double)metric_elem(v[j], cn, row0 + k + 32 * j);
    }
    for (; k < K; k += 32) s += (double)metric_elem(p[(int64_t)k * D], cn, row0 + k);
  }
  part[w][lane] = s;
  __syncthreads();
  if (w == 0 && d < D) {
    double t = 0.0;
#pragma unroll 1
    for (int j = 0; j < 32; ++j) t += part[j][lane];
    m[(int64_t)b * D + d] = (float)(t / (double)K);
  }
}

// v split into three 16-bit parts whose weighted sum is v to about 24 bits:
// bf16 parts are successive residuals (weights 1, 1, 1); fp16 parts are scaled
// by 2^-15, 2^-4, 2^7 (weights 2^15, 2^4, 2^-7) so |v| up to 2^31 stays in
// range.  Parts below the type's smallest normal are flushed to zero so no
// operand is subnormal.
__device__ __forceinline__ void bias_parts(double v, bool f16, uint16_t out[3]) {
  if (!f16) {
    double r = v;
    for (int i = 0; i < 3; ++i) {
      __nv_bfloat16 q = __double2bfloat16(r);
      float qf = __bfloat162float(q);
      if (fabsf(qf) < 1.17549435e-38f) { q = __float2bfloat16_rn(0.0f); qf = 0.0f; }
      out[i] = __bfloat16_as_ushort(q);
      r -= (double)qf;
    }
  } else {
    const double scale[3] = {1.0 / 32768.0, 1.0 / 16.0, 128.0};   // 1 / weight
    double r = v;
    for (int i = 0; i < 3; ++i) {
      double t = r * scale[i];
      t = fmin(fmax(t, -65504.0), 65504.0);
      __half q = __double2half(t);
      float qf = __half2float(q);
      if (fabsf(qf) < 6.1035156e-5f) { q = __float2half_rn(0.0f); qf = 0.0f; }
      out[i] = __half_as_ushort(q);
      r -= (double)qf / scale[i];
    }
  }
}

// q(v) in the points' 16-bit type, as raw bits and as the value it rounds to
__device__ __forceinline__ uint16_t q16(float v, bool bf, float* back) {
  if (bf) {
    const __nv_bfloat16 q = __float2bfloat16_rn(v);
    *back = __bfloat162float(q);
    return __bfloat16_as_ushort(q);
  }
  const __half q = __float2half_rn(v);
  *back = __half2float(q);
  return __half_as_ushort(q);
}

// Four padded centroid rows per warp, eight lanes per row; each lane takes
// four consecutive elements at a time (D is a multiple of 4 for every dtype:
// the rows of x are 16-byte multiples).
__global__ void prep_centroids_kernel(const float* __restrict__ c, const float* __restrict__ m,
                                      int B, int K, int Kp, int D, int dtype,
                                      void* __restrict__ cq, uint16_t* __restrict__ caug,
                                      const double* __restrict__ cn, bool bias) {
  const int lane = threadIdx.x & 31, l8 = lane & 7;
  const int64_t row =
      ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4 + (lane >> 3);
  const bool valid = row < (int64_t)B * Kp;
  const int b = valid ? (int)(row / Kp) : 0, k = valid ? (int)(row % Kp) : 0;
  const bool real = valid && k < K;
  const float* src = c + ((int64_t)b * K + k) * D;
  const float* mb = m + (int64_t)b * D;
  double acc = 0.0;
  if (dtype == FKM_F32) {
    const int Dp = (D + 7) & ~7;
    uint16_t* out = static_cast<uint16_t*>(cq) + row * (int64_t)(2 * Dp);
    for (int d = 4 * l8; valid && d < D; d += 32) {
      const float4 mm = *reinterpret_cast<const float4*>(mb + d);
      float4 cv = real ? *reinterpret_cast<const float4*>(src + d) : mm;
      if (real && cn) {
        const int64_t r = (int64_t)b * K + k;
        cv = make_float4(metric_elem(cv.x, cn, r), metric_elem(cv.y, cn, r),
                         metric_elem(cv.z, cn, r), metric_elem(cv.w, cn, r));
      }
      const float v[4] = {cv.x - mm.x, cv.y - mm.y, cv.z - mm.z, cv.w - mm.w};
      const float mv[4] = {mm.x, mm.y, mm.z, mm.w};
      uint16_t hb[4], lb[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float hf, lf;
        hb[j] = q16(v[j], true, &hf);
        lb[j] = q16(v[j] - hf, true, &lf);
        acc += (double)v[j] * ((double)v[j] + 2.0 * (double)mv[j]);
      }
      *reinterpret_cast<uint2*>(out + d) =
          make_uint2(hb[0] | ((uint32_t)hb[1] << 16), hb[2] | ((uint32_t)hb[3] << 16));
      *reinterpret_cast<uint2*>(out + Dp + d) =
          make_uint2(lb[0] | ((uint32_t)lb[1] << 16), lb[2] | ((uint32_t)lb[3] << 16));
    }
  } else {
    const bool bf = dtype == FKM_BF16;
    uint16_t* out = static_cast<uint16_t*>(cq) + row * (int64_t)D;
    for (int d = 4 * l8; valid && d < D; d += 32) {
      const float4 mm = *reinterpret_cast<const float4*>(mb + d);
      float4 cv = real ? *reinterpret_cast<const float4*>(src + d) : mm;
      if (real && cn) {
        const int64_t r = (int64_t)b * K + k;
        cv = make_float4(metric_elem(cv.x, cn, r), metric_elem(cv.y, cn, r),
                         metric_elem(cv.z, cn, r), metric_elem(cv.w, cn, r));
      }
      const float v[4] = {cv.x - mm.x, cv.y - mm.y, cv.z - mm.z, cv.w - mm.w};
      const float mv[4] = {mm.x, mm.y, mm.z, mm.w};
      uint16_t qb[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float f;
        qb[j] = q16(v[j], bf, &f);
        acc += (double)f * ((double)f + 2.0 * (double)mv[j]);
      }
      *reinterpret_cast<uint2*>(out + d) =
          make_uint2(qb[0] | ((uint32_t)qb[1] << 16), qb[2] | ((uint32_t)qb[3] << 16));
    }
  }
  // sum over the row's eight lanes; the butterfly leaves every lane the same
  // value (each level adds the same two operands on both sides)
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  // the bias slab: [-n/2 in three parts, 0 x 13]; padding rows are all zero
  // (the assign kernel masks their columns); lane l8 writes entries 2 l8, 2 l8 + 1
  uint16_t parts[3] = {0, 0, 0};
  if (real && bias) bias_parts(-0.5 * acc, dtype == FKM_F16, parts);
  if (valid) {
    const int e = 2 * l8;
    const uint32_t lo = e == 0 ? parts[0] : e == 2 ? parts[2] : 0u;
    const uint32_t hi = e == 0 ? parts[1] : 0u;
    *reinterpret_cast<uint32_t*>(caug + row * AUG_SLAB + e) = lo | (hi << 16);
  }
}

// one warp per point row; xn[row] = ||x - m[batch]||^2 when m is given
__global__ void points_prep_kernel(const void* __restrict__ x, int64_t rows, int D, int dtype,
                                   __nv_bfloat16* __restrict__ xs, float* __restrict__ xn,
                                   const float* __restrict__ m, int N) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  double acc = 0.0;
  const float* mb = m ? m + (row / N) * D : nullptr;
  if (dtype == FKM_F32) {
    const int Dp = (D + 7) & ~7;
    const float* src = static_cast<const float*>(x) + row * D;
    __nv_bfloat16* out = xs + row * (int64_t)(2 * Dp);
    for (int d = lane; d < D; d += 32) {
      float v = src[d];
      __nv_bfloat16 h = __float2bfloat16_rn(v);
      __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
      if (xs) {
        out[d] = h;
        out[Dp + d] = l;
      }
      const double dv = (double)v - (mb ? (double)mb[d] : 0.0);
      acc += dv * dv;
    }
  } else {
    // 16-bit points: 8-byte loads, four values per lane per step
    const uint2* src = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(x) + row * D);
    const int nv = D / 4;
    for (int v = lane; v < nv; v += 32) {
      uint2 w = src[v];
      uint32_t wd[2] = {w.x, w.y};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float a, bb;
        if (dtype == FKM_BF16) {
          a = __uint_as_float(wd[h] << 16);
          bb = __uint_as_float(wd[h] & 0xFFFF0000u);
        } else {
          __half2 hv = *reinterpret_cast<__half2*>(&wd[h]);
          float2 f = __half22float2(hv);
          a = f.x;
          bb = f.y;
        }
        const double da = (double)a - (mb ? (double)mb[4 * v + 2 * h] : 0.0);
        const double db = (double)bb - (mb ? (double)mb[4 * v + 2 * h + 1] : 0.0);
        acc += da * da + db * db;
      }
    }
  }
  acc = warp_sum(acc);
  if (lane == 0 && xn) xn[row] = (float)acc;
}

}  // namespace

fkm_status launch_prep_centroids(const float* centers, int B, int K, int Kp, int D, int dtype,
                                 float* m, void* cq, void* caug, cudaStream_t st, int metric,
                                 double* cnorm) {
  const double* cn = nullptr;
  if (metric == FKM_METRIC_COSINE) {
    const int64_t rows = (int64_t)B * K;
    row_norms_kernel<<<(unsigned)ceil_div(rows, 8), 256, 0, st>>>(centers, rows, D, cnorm);
    note_launch();
    cn = cnorm;
  }
  center_kernel<<<dim3((unsigned)B, (unsigned)ceil_div(D, 32)), 1024, 0, st>>>(centers, B, K, D,
                                                                              m, cn);
  const int64_t rows = (int64_t)B * Kp;
  const int wpb = 8;   // 4 rows per warp
  prep_centroids_kernel<<<(unsigned)ceil_div(rows, 4 * wpb), wpb * 32, 0, st>>>(
      centers, m, B, K, Kp, D, dtype, cq, static_cast<uint16_t*>(caug), cn,
      metric == FKM_METRIC_EUCLID);
  note_launch(2);
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

fkm_status launch_points_prep(const void* x, int64_t rows, int D, int dtype, void* xs, float* xn,
                              cudaStream_t st, const float* m, int N) {
  if (rows == 0) return FKM_OK;
  const int wpb = 8;
  points_prep_kernel<<<(unsigned)ceil_div(rows, wpb), wpb * 32, 0, st>>>(
      x, rows, D, dtype, static_cast<__nv_bfloat16*>(xs), xn, m, N > 0 ? N : 1);
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

}  // namespace fkm
