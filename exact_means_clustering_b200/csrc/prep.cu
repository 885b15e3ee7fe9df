// Operand preparation for the assign kernel.
//
//  center: per batch the mean centroid m (fp64 sum over k in a fixed order,
//    divided by K, rounded to fp32).  The assignment works on offsets from m:
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
#include "ptx_sm100.cuh"

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
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
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

// m[b][d] = fp32(S / K), S summed in fp64 in one fixed order that does not
// depend on the launch (the fused end-of-iteration kernel below follows the
// same order, so both give m bit for bit): the padded rows [0, Kp) are cut
// into MEAN_CHUNKS contiguous chunks of R = Kp / MEAN_CHUNKS rows; partial
// (r, w) of chunk r sums the rows r*R + w, r*R + w + MEAN_WAYS, ... below K in
// ascending order; a chunk adds its partials in order w = 0, 1, ..., and S
// adds the chunks in order r = 0, 1, ....  Grid (B, 32-dimension groups,
// MEAN_CHUNKS), one cluster of MEAN_CHUNKS CTAs per (batch, group): CTA r
// forms chunk r, warp w partial (r, w) for the 32 dimensions of its lanes
// (coalesced rows, eight rows' loads in flight), and CTA 0 adds the chunks
// from distributed shared memory.
__global__ void __cluster_dims__(1, 1, MEAN_CHUNKS) __launch_bounds__(MEAN_WAYS * 32)
    center_kernel(const float* __restrict__ c, int B, int K, int Kp, int D,
                  float* __restrict__ m, const double* __restrict__ cn) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  __shared__ double part[MEAN_WAYS][33];
  __shared__ double chunk[32];
  const int b = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int r = (int)ptx::cluster_ctarank();   // == blockIdx.z
  const int d = blockIdx.y * 32 + lane;
  const int R = Kp / MEAN_CHUNKS;
  double s = 0.0;
  if (d < D) {
    const float* p = c + (int64_t)b * K * D + d;
    const int64_t row0 = (int64_t)b * K;
    const int k0 = r * R + w;
    int i = 0;
    for (; i + 7 * MEAN_WAYS < R; i += 8 * MEAN_WAYS) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = k0 + i + j * MEAN_WAYS;
        v[j] = k < K ? p[(int64_t)k * D] : 0.0f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = k0 + i + j * MEAN_WAYS;
        if (k < K) s += (double)metric_elem(v[j], cn, row0 + k);
      }
    }
    for (; i < R; i += MEAN_WAYS) {
      const int k = k0 + i;
      if (k < K) s += (double)metric_elem(p[(int64_t)k * D], cn, row0 + k);
    }
  }
  part[w][lane] = s;
  __syncthreads();
  if (w == 0) {
    double t = 0.0;
#pragma unroll 1
    for (int q = 0; q < MEAN_WAYS; ++q) t += part[q][lane];
    chunk[lane] = t;
  }
  ptx::cluster_sync();   // every chunk's sums visible across the cluster
  if (r == 0 && w == 0 && d < D) {
    double t = 0.0;
#pragma unroll 1
    for (int q = 0; q < MEAN_CHUNKS; ++q)
      t += ptx::ld_shared_cluster_f64(ptx::mapa_rank(&chunk[lane], q));
    m[(int64_t)b * D + d] = (float)(t / (double)K);
  }
  ptx::cluster_sync();   // no CTA leaves while CTA 0 still reads its shared memory
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

// One padded centroid row, eight lanes per row (l8 = lane & 7); each lane
// takes four consecutive elements at a time (D is a multiple of 4 for every
// dtype: the rows of x are 16-byte multiples).  src: the fp32 centroid row
// (read only when real), mb: the batch's mean centroid, crow: the row's index
// b*K + k (cosine norms), row: its index b*Kp + k in the operands.  Every lane
// of the warp calls this (the row's lanes exchange partial sums).
__device__ __forceinline__ void prep_row(const float* __restrict__ src,
                                         const float* __restrict__ mb, bool valid, bool real,
                                         int64_t crow, int64_t row, int D, int dtype,
                                         void* __restrict__ cq, uint16_t* __restrict__ caug,
                                         const double* __restrict__ cn, bool bias, int l8) {
  double acc = 0.0;
  if (dtype == FKM_F32) {
    const int Dp = (D + 7) & ~7;
    uint16_t* out = static_cast<uint16_t*>(cq) + row * (int64_t)(2 * Dp);
    for (int d = 4 * l8; valid && d < D; d += 32) {
      const float4 mm = *reinterpret_cast<const float4*>(mb + d);
      float4 cv = real ? *reinterpret_cast<const float4*>(src + d) : mm;
      if (real && cn)
        cv = make_float4(metric_elem(cv.x, cn, crow), metric_elem(cv.y, cn, crow),
                         metric_elem(cv.z, cn, crow), metric_elem(cv.w, cn, crow));
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
      if (real && cn)
        cv = make_float4(metric_elem(cv.x, cn, crow), metric_elem(cv.y, cn, crow),
                         metric_elem(cv.z, cn, crow), metric_elem(cv.w, cn, crow));
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

// Four padded centroid rows per warp.
__global__ void prep_centroids_kernel(const float* __restrict__ c, const float* __restrict__ m,
                                      int B, int K, int Kp, int D, int dtype,
                                      void* __restrict__ cq, uint16_t* __restrict__ caug,
                                      const double* __restrict__ cn, bool bias) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t row =
      ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 4 + (lane >> 3);
  const bool valid = row < (int64_t)B * Kp;
  const int b = valid ? (int)(row / Kp) : 0, k = valid ? (int)(row % Kp) : 0;
  const bool real = valid && k < K;
  prep_row(c + ((int64_t)b * K + k) * D, m + (int64_t)b * D, valid, real, (int64_t)b * K + k,
           row, D, dtype, cq, caug, cn, bias, lane & 7);
}

// The end of a Lloyd iteration in one launch: one thread-block cluster of
// MEAN_CHUNKS CTAs per batch (grid MEAN_CHUNKS x B), CTA r owning the padded
// rows [r R, (r+1) R), R = Kp / MEAN_CHUNKS.
//   1. finalize (as finalize_kernel, or finalize_sim_kernel for dot and
//      cosine k-means): warp w takes the rows r R + w, r R + w + MEAN_WAYS,
//      ...: count, new centroid (s/n of a crossing run, the value the segment
//      sums wrote for an interior one, the previous centroid for an empty
//      cluster), its shift, and the running fp64 sums of the new centroid's
//      columns (as the assignment sees them) -- partial (r, w) of the mean's
//      order;
//   2. the CTA adds its partials (w = 0, 1, ...), the cluster barrier makes
//      every CTA's sums visible, and every CTA adds the chunks (r = 0, 1, ...)
//      from distributed shared memory: m, bit for bit center_kernel's; CTA 0
//      also writes m, the batch's shift and, for dot and cosine, its
//      objective (same chunked order);
//   3. the CTA prepares the operands of its rows (prep_row) against m.
// Columns are held four per lane, so D <= FP_MAX_D (128 for dot and cosine).
constexpr int FP_WARPS = MEAN_WAYS;
constexpr int FP_MAX_D = 256;

struct FinPrepParams {
  int B, K, Kp, D, dtype, range;
  const int32_t* segstart;
  const int32_t* segend;
  double* sums64;      // crossing runs' fp64 sums, zeroed after use
  const float* prev;
  float* centers;
  int32_t* counts;
  float* m;
  void* cq;
  uint16_t* caug;
  double* shift_out;   // optional [B]
  double* max_shift;   // optional (zeroed by the caller): max over batches
  int metric;          // FKM_METRIC_*; dot and cosine need D <= 128
  double* cnorm;       // cosine: the new centroids' row norms [B*K]
  double* obj_out;     // dot / cosine, optional [B]: the objective of the assignment
};

// One cluster of the dot / cosine finalize (finalize_sim_kernel's arithmetic
// for D <= 128, one 16-byte piece per lane): writes the new centroid (the
// mean, its unit direction for cosine, or prev for an empty or zero-sum
// cluster) and the count; returns the shift in every lane and adds the
// cluster's objective share to *obj; cs receives the column values the mean
// centroid adds (the row scaled by its norm for cosine, whose norm, summed
// in row_norms_kernel's order, goes to cnorm).
__device__ __forceinline__ double finalize_sim_row(const FinPrepParams& p, int64_t key,
                                                   int32_t nk, bool interior, int lane,
                                                   double* obj, double (&cs)[4]) {
  const bool cosine = p.metric == FKM_METRIC_COSINE;
  const int d = 4 * lane;
  const bool on = d < p.D;
  const int64_t e = key * p.D + d;
  const double n = (double)nk;
  float4 pv = make_float4(0.f, 0.f, 0.f, 0.f), v = pv;
  double sd[4] = {0.0, 0.0, 0.0, 0.0};
  if (on) {
    pv = *reinterpret_cast<const float4*>(p.prev + e);
    if (nk > 0 && interior) {
      v = *reinterpret_cast<const float4*>(p.centers + e);
      sd[0] = (double)v.x * n;
      sd[1] = (double)v.y * n;
      sd[2] = (double)v.z * n;
      sd[3] = (double)v.w * n;
    } else if (nk > 0) {
      double2* s2 = reinterpret_cast<double2*>(p.sums64 + e);
      const double2 a = s2[0], c = s2[1];
      sd[0] = a.x;
      sd[1] = a.y;
      sd[2] = c.x;
      sd[3] = c.y;
      v = make_float4((float)(a.x / n), (float)(a.y / n), (float)(c.x / n), (float)(c.y / n));
      s2[0] = make_double2(0.0, 0.0);
      s2[1] = make_double2(0.0, 0.0);
    }
  }
  const float vv4[4] = {v.x, v.y, v.z, v.w}, pv4[4] = {pv.x, pv.y, pv.z, pv.w};
  double vv = 0.0, pp = 0.0, sp = 0.0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    vv += (double)vv4[j] * (double)vv4[j];
    pp += (double)pv4[j] * (double)pv4[j];
    sp += sd[j] * (double)pv4[j];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vv += __shfl_xor_sync(0xffffffffu, vv, o);
    pp += __shfl_xor_sync(0xffffffffu, pp, o);
    sp += __shfl_xor_sync(0xffffffffu, sp, o);
  }
  const double pn = sqrt(pp), vn = sqrt(vv);
  const bool keep = nk == 0 || (cosine && !(vv > 0.0));
  float o4[4];
  double sh = 0.0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    o4[j] = keep ? pv4[j] : cosine ? (float)((double)vv4[j] / vn) : vv4[j];
    const double df = (double)o4[j] - (double)pv4[j];
    sh += df * df;
  }
  if (on) *reinterpret_cast<float4*>(p.centers + e) = make_float4(o4[0], o4[1], o4[2], o4[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sh += __shfl_xor_sync(0xffffffffu, sh, o);
  *obj += cosine ? (pn > 0.0 ? sp / pn : 0.0) : sp;
  if (lane == 0 && p.counts) p.counts[key] = nk;
  if (!cosine) {
#pragma unroll
    for (int j = 0; j < 4; ++j) cs[j] += on ? (double)o4[j] : 0.0;
    return sh;
  }
  // ||o|| in row_norms_kernel's order: lane l sums elements l, l + 32, ...,
  // which lanes (l + 32 q) / 4 hold as their component l % 4
  double s = 0.0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int src = (lane >> 2) + 8 * q;
    float t[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) t[j] = __shfl_sync(0xffffffffu, o4[j], src);
    const float ov = t[lane & 3];
    if (lane + 32 * q < p.D) s += (double)ov * (double)ov;
  }
  s = warp_sum(s);
  const double cn = sqrt(s);
  if (lane == 0) p.cnorm[key] = cn;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    cs[j] += on ? (double)(cn > 0.0 ? (float)((double)o4[j] / cn) : 0.0f) : 0.0;
  return sh;
}

template <bool kEuclid>
__global__ void __cluster_dims__(MEAN_CHUNKS, 1, 1) __launch_bounds__(FP_WARPS * 32, 2)
    finalize_prep_kernel(FinPrepParams p) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  __shared__ double colsum[FP_WARPS][FP_MAX_D];
  __shared__ double cta_sum[FP_MAX_D];
  __shared__ double wshift[FP_WARPS];
  __shared__ double wobj[FP_WARPS];
  __shared__ double cta_shift;
  __shared__ double cta_obj;
  __shared__ __align__(16) float msh[FP_MAX_D];
  const int r = (int)ptx::cluster_ctarank();
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = p.Kp / MEAN_CHUNKS;
  const int D = p.D;
  const int64_t kb = (int64_t)b * p.K;

  // ---- 1. finalize this CTA's rows
  constexpr int J = FP_MAX_D / 128;   // four-column pieces per lane
  double cs[J][4];
#pragma unroll
  for (int j = 0; j < J; ++j) cs[j][0] = cs[j][1] = cs[j][2] = cs[j][3] = 0.0;
  double shw = 0.0, objw = 0.0;
  constexpr bool euclid = kEuclid;   // else dot / cosine (p.metric)
  // the next row's segment bounds are loaded while the current row is
  // finalized, so each row waits for one round trip to memory, not two
  const int kend = min(r * R + R, p.K);
  int32_t nb0 = 0, nb1 = 0;
  if (r * R + warp < kend) {
    nb0 = p.segstart[kb + r * R + warp];
    nb1 = p.segend[kb + r * R + warp];
  }
  for (int k = r * R + warp; k < kend; k += FP_WARPS) {
    const int64_t key = kb + k;
    const int32_t s0 = nb0, s1 = nb1;
    if (k + FP_WARPS < kend) {
      nb0 = p.segstart[key + FP_WARPS];
      nb1 = p.segend[key + FP_WARPS];
    }
    const int32_t nk = s1 - s0;
    const bool interior = nk > 0 && (s0 / p.range) == ((s1 - 1) / p.range);
    if constexpr (!euclid) {
      shw += finalize_sim_row(p, key, nk, interior, lane, &objw, cs[0]);
      continue;
    }
    if (lane == 0 && p.counts) p.counts[key] = nk;
    double sh = 0.0;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int d = 4 * lane + 128 * j;
      if (d >= D) break;
      const int64_t e = key * D + d;
      const float4 pv = *reinterpret_cast<const float4*>(p.prev + e);
      float4 v;
      if (nk == 0) {
        v = pv;
      } else if (interior) {
        v = *reinterpret_cast<const float4*>(p.centers + e);
      } else {
        double2* s2 = reinterpret_cast<double2*>(p.sums64 + e);
        const double2 a = s2[0], c = s2[1];
        const double n = (double)nk;
        v = make_float4((float)(a.x / n), (float)(a.y / n), (float)(c.x / n), (float)(c.y / n));
        s2[0] = make_double2(0.0, 0.0);
        s2[1] = make_double2(0.0, 0.0);
      }
      *reinterpret_cast<float4*>(p.centers + e) = v;
      const double d0 = (double)v.x - (double)pv.x, d1 = (double)v.y - (double)pv.y;
      const double d2 = (double)v.z - (double)pv.z, d3 = (double)v.w - (double)pv.w;
      sh += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
      cs[j][0] += (double)v.x;
      cs[j][1] += (double)v.y;
      cs[j][2] += (double)v.z;
      cs[j][3] += (double)v.w;
    }
    shw += warp_sum(sh);   // the same value in every lane
  }
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int d = 4 * lane + 128 * j;
    if (d < D) {
      colsum[warp][d] = cs[j][0];
      colsum[warp][d + 1] = cs[j][1];
      colsum[warp][d + 2] = cs[j][2];
      colsum[warp][d + 3] = cs[j][3];
    }
  }
  if (lane == 0) {
    wshift[warp] = shw;
    wobj[warp] = objw;
  }
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double t = 0.0;
#pragma unroll 1
    for (int w = 0; w < FP_WARPS; ++w) t += colsum[w][d];
    cta_sum[d] = t;
  }
  if (threadIdx.x == 0) {
    double t = 0.0, o = 0.0;
#pragma unroll 1
    for (int w = 0; w < FP_WARPS; ++w) {
      t += wshift[w];
      o += wobj[w];
    }
    cta_shift = t;
    cta_obj = o;
  }
  // ---- 2. the batch's mean and shift across the cluster
  ptx::cluster_sync();   // release / acquire: every CTA's sums (and centroids) visible
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double t = 0.0;
#pragma unroll 1
    for (int q = 0; q < MEAN_CHUNKS; ++q)
      t += ptx::ld_shared_cluster_f64(ptx::mapa_rank(&cta_sum[d], q));
    msh[d] = (float)(t / (double)p.K);
    if (r == 0) p.m[(int64_t)b * D + d] = msh[d];
  }
  if (r == 0 && threadIdx.x == 0) {
    double t = 0.0;
#pragma unroll 1
    for (int q = 0; q < MEAN_CHUNKS; ++q)
      t += ptx::ld_shared_cluster_f64(ptx::mapa_rank(&cta_shift, q));
    if (p.shift_out) p.shift_out[b] = t;
    if (p.max_shift)   // shift >= 0: the bit pattern orders like the value
      atomicMax(reinterpret_cast<unsigned long long*>(p.max_shift),
                (unsigned long long)__double_as_longlong(t));
    if (!euclid && p.obj_out) {
      double o = 0.0;
#pragma unroll 1
      for (int q = 0; q < MEAN_CHUNKS; ++q)
        o += ptx::ld_shared_cluster_f64(ptx::mapa_rank(&cta_obj, q));
      p.obj_out[b] = o;
    }
  }
  ptx::cluster_sync();   // no CTA leaves while another still reads its shared memory
  // ---- 3. the next assign's operands for this CTA's rows
  for (int i = warp * 4 + (lane >> 3); i < R; i += FP_WARPS * 4) {
    const int k = r * R + i;
    const bool real = k < p.K;
    prep_row(p.centers + (kb + k) * D, msh, true, real, kb + k, (int64_t)b * p.Kp + k, D,
             p.dtype, p.cq, p.caug, p.metric == FKM_METRIC_COSINE ? p.cnorm : nullptr, euclid,
             lane & 7);
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
    FKM_CUDA_TRY(launch_pdl(row_norms_kernel, dim3((unsigned)ceil_div(rows, 8)), dim3(256), 0, st,
                            centers, rows, D, cnorm));
    note_launch();
    cn = cnorm;
  }
  FKM_CUDA_TRY(launch_pdl(center_kernel, dim3((unsigned)B, (unsigned)ceil_div(D, 32), MEAN_CHUNKS),
                          dim3(MEAN_WAYS * 32), 0, st, centers, B, K, Kp, D, m, cn));
  const int64_t rows = (int64_t)B * Kp;
  const int wpb = 8;   // 4 rows per warp
  FKM_CUDA_TRY(launch_pdl(prep_centroids_kernel, dim3((unsigned)ceil_div(rows, 4 * wpb)),
                          dim3(wpb * 32), 0, st, centers, m, B, K, Kp, D, dtype, cq,
                          static_cast<uint16_t*>(caug), cn, metric == FKM_METRIC_EUCLID));
  note_launch(2);
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

// A CTA finalizes and prepares Kp / MEAN_CHUNKS rows, one after another per
// warp; beyond 128 rows (Kp > 1024) the separate kernels, with every row
// in its own warp, finish sooner.
bool finalize_prep_fits(int B, int Kp, int D, int metric) {
  return D <= (metric == FKM_METRIC_EUCLID ? FP_MAX_D : 128) && B <= 65535 && Kp <= 1024;
}

fkm_status launch_finalize_prep(int B, int K, int Kp, int D, int dtype, int range,
                                const int32_t* segstart, const int32_t* segend, double* sums64,
                                const float* prev, float* centers, int32_t* counts, float* m,
                                void* cq, void* caug, double* shift_out, double* max_shift,
                                cudaStream_t st, int metric, double* cnorm, double* obj_out) {
  if (!finalize_prep_fits(B, Kp, D, metric) || Kp % BN != 0 ||
      (metric == FKM_METRIC_COSINE && !cnorm)) {
    set_error("finalize_prep: D = %d or Kp = %d out of range", D, Kp);
    return FKM_ERR_INTERNAL;
  }
  FinPrepParams p;
  p.B = B;
  p.K = K;
  p.Kp = Kp;
  p.D = D;
  p.dtype = dtype;
  p.range = range;
  p.segstart = segstart;
  p.segend = segend;
  p.sums64 = sums64;
  p.prev = prev;
  p.centers = centers;
  p.counts = counts;
  p.m = m;
  p.cq = cq;
  p.caug = static_cast<uint16_t*>(caug);
  p.shift_out = shift_out;
  p.max_shift = max_shift;
  p.metric = metric;
  p.cnorm = cnorm;
  p.obj_out = obj_out;
  if (metric == FKM_METRIC_EUCLID)
    FKM_CUDA_TRY(launch_pdl(finalize_prep_kernel<true>, dim3(MEAN_CHUNKS, (unsigned)B),
                            dim3(FP_WARPS * 32), 0, st, p));
  else
    FKM_CUDA_TRY(launch_pdl(finalize_prep_kernel<false>, dim3(MEAN_CHUNKS, (unsigned)B),
                            dim3(FP_WARPS * 32), 0, st, p));
  note_launch();
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
