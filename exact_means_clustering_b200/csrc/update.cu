// Sort-Inverse Update, after the argsort ("Flash-KMeans：快速且内存高效精确K-Means
// 聚类" summary, section 方法步骤详情 step (2); "Flash-KMeans: Fast and
// Memory-Efficient Exact K-Means" summary, section "Method"):
//
//   bounds      runs of equal keys in the sorted order: start/end per key, so
//               counts = end - start are exact integers (from the counting
//               sort's scan, or written by segsum from its staged keys).
//   segsum      the sorted order is cut into ranges of SEG_RANGE rows, one warp
//               per range.  The warp walks its rows in order, gathering each
//               row of the UNPERMUTED x by the sorted index with 16-byte loads
//               (several rows per warp step when a row is narrower than 512 B)
//               and adding it into fp64 registers.  When the key changes the
//               partial sum is reduced across the warp with shuffles and
//               flushed once: a run that lies inside this range is final, so
//               the warp writes its centroid s/n directly; a run that crosses a
//               range boundary is added to fp64 sums with one atomic per
//               element (at most two such flushes per range), i.e. the pages'
//               one atomic_add per segment boundary, O(K + N/B_N) of them.
//               The same pass forms the objective of the assignment,
//               sum ||x - c_hat||^2 with the direct difference (c_hat = the
//               centroid the assign step measured against), so the reported
//               inertia does not suffer the cancellation of the expanded form.
//   finalize    per cluster: counts, c = s/n for crossing runs, the previous
//               centroid for empty clusters (a reading: the pages give only
//               c = s/n), and the shift ||c_new - c_old||^2.
//   batch_reduce  per batch, in fixed order: shift = sum_k shift_k.
// Inside the Lloyd loop, for D <= 256 and Kp <= 1024, finalize and the batch
// shifts run fused with the next assign's operand preparation
// (finalize_prep_kernel, prep.cu).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fkm_internal.cuh"

namespace fkm {
namespace {

// Rows longer than 512 bytes are summed in slabs of columns, one launch per
// slab: x, centers, sums64, the centroid rows and the mean point at the slab's
// first column, D its width, Dfull the whole row length.
struct SegParams {
  const void* x;
  const int32_t* skeys;
  const int32_t* svals;
  int64_t n;
  int D;                 // columns in this slab
  int Dfull;             // columns of a whole row (stride of centers / sums / centroid rows)
  int BK;
  int64_t row_bytes;     // bytes between rows of x
  int ebytes;            // bytes per element of x
  int V;                 // 16-byte vectors per slab row
  int range;             // sorted rows per warp (<= SEG_RANGE)
  double* sums64;
  float* centers;
  bool accumulate_all;   // out-of-core chunks: every run goes to sums64
  ObjArgs oa;
  unsigned long long* atomics;   // optional: count of fp64 atomic additions to sums64
  int32_t* segstart;   // optional (cleared to zero by the caller): run bounds per key,
  int32_t* segend;     // written here from the staged keys
  int* status;         // checked build: out-of-range row indices are reported here
};

// 16-byte vectors of the storage type, widened to float.
template <int DT> struct Vec;
template <> struct Vec<FKM_BF16> {
  static constexpr int E = 8;
  __device__ static void widen2(const uint4& v, float2* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  }
  __device__ static void widen(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};
template <> struct Vec<FKM_F16> {
  static constexpr int E = 8;
  __device__ static void widen2(const uint4& v, float2* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
  }
  __device__ static void widen(const uint4& v, float* f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <> struct Vec<FKM_F32> {
  static constexpr int E = 4;
  __device__ static void widen2(const uint4& v, float2* f) {
    f[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    f[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
  __device__ static void widen(const uint4& v, float* f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
};

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Flush of one run (its fp32 partials already folded into acc): the
// partials are summed over the row groups (xor shuffles), and group 0 writes
// either the final centroid (run inside this range, nk rows) or adds to the
// fp64 accumulators (run crossing a range boundary).
template <int E, int LPR>
__device__ __forceinline__ void flush_run(const SegParams& p, int key, int g, int sub,
                                          bool lane_has_vec, bool interior, int nk,
                                          double (&acc)[E]) {
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  if (g == 0 && lane_has_vec) {
    const int64_t col0 = (int64_t)sub * E;
    if (interior) {
      // one fp64 reciprocal per run (its error, below 2^-52 relative, is
      // far below the fp32 rounding that follows)
      const double rn = 1.0 / (double)nk;
      float* c = p.centers + (int64_t)key * p.Dfull + col0;
      if (col0 + E <= p.D && (E & 3) == 0) {
        // whole 16-byte pieces (row starts and col0 are 16-byte aligned)
#pragma unroll
        for (int e = 0; e < E; e += 4)
          *reinterpret_cast<float4*>(c + e) =
              make_float4((float)(acc[e] * rn), (float)(acc[e + 1] * rn),
                          (float)(acc[e + 2] * rn), (float)(acc[e + 3] * rn));
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e)
          if (col0 + e < p.D) c[e] = (float)(acc[e] * rn);
      }
    } else {
      double* sd = p.sums64 + (int64_t)key * p.Dfull + col0;
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (col0 + e < p.D) atomicAdd(sd + e, acc[e]);
      // instrumentation: this flush made p.D element atomics in all
      if (sub == 0 && p.atomics) atomicAdd(p.atomics, (unsigned long long)p.D);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.0;
}

#ifndef FKM_SEG_STAGES
#define FKM_SEG_STAGES 4
#endif
#ifndef FKM_SEG_MIN_BLOCKS
#define FKM_SEG_MIN_BLOCKS 3
#endif
constexpr int SEG_WARPS = 8;                // warps (ranges) per block
constexpr int SEG_STAGES = FKM_SEG_STAGES;  // row-gather steps in flight per warp
static_assert((SEG_STAGES & (SEG_STAGES - 1)) == 0, "the ring index is a mask");


// Per-warp shared memory: the range's (key, row) pairs, the start position of
// every run (plus an end sentinel), and the gather ring.
struct SegWarpSmem {
  int2 kv[SEG_RANGE + 1];   // + a (-1, 0) sentinel read by gathers past the range
  uint4 ring[SEG_STAGES][32];
  double2 acc[4][32];   // per lane fp64 sums of its vector: [element pair][lane]
  int16_t runs[SEG_RANGE + 1];
};
constexpr size_t SEG_SMEM_BYTES = sizeof(SegWarpSmem) * SEG_WARPS;

__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gmem),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_stages() {
  asm volatile("cp.async.wait_group %0;" ::"n"(SEG_STAGES - 1) : "memory");
}

// One warp per SEG_RANGE sorted rows.  The range's (key, row) pairs are
// staged in shared memory first, together with the start of every run of
// equal keys and the keys just outside the range, so a run's length and
// whether it crosses the range boundary are known without touching global
// memory.  Then every lane gathers its 16-byte piece of the rows RPS at a
// time (LPR = 32 / RPS lanes per row, lane `sub` holding vector `sub` of its
// row) with cp.async into a per-warp ring of SEG_STAGES steps, so
// SEG_STAGES * RPS rows are in flight while the warp adds the oldest step.
// Rows are added in fp32 and folded into fp64 at every run flush and every 16
// steps.  For the objective, the centroid row of the next run is loaded when
// the current run starts, so it has arrived by the time it is needed.
template <int DT, int RPS>
__global__ void __launch_bounds__(SEG_WARPS * 32, FKM_SEG_MIN_BLOCKS)
    segsum_kernel(SegParams p) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  constexpr int E = Vec<DT>::E;
  constexpr int LPR = 32 / RPS;
  extern __shared__ __align__(16) uint8_t seg_smem[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  SegWarpSmem& ws = reinterpret_cast<SegWarpSmem*>(seg_smem)[wid];
  const int g = lane / LPR, sub = lane % LPR;
  const bool lane_has_vec = sub < p.V;
  const bool want_obj = p.oa.obj != nullptr;
  const int64_t elem_bytes_ = p.ebytes;
  const int64_t r = (int64_t)blockIdx.x * SEG_WARPS + wid;
  const int64_t nranges = ceil_div(p.n, p.range);
  if (r >= nranges) return;
  const int64_t j0 = r * p.range;
  const int nrows = (int)((j0 + p.range < p.n) ? p.range : p.n - j0);

  // ---- staging: all loads first, then the stores
  int2 e_[SEG_RANGE / 32];
#pragma unroll
  for (int t = 0; t < SEG_RANGE / 32; ++t) {
    const int i = t * 32 + lane;
    e_[t] = make_int2(-1, 0);
    if (i < nrows) {
      e_[t].x = p.skeys[j0 + i];
      e_[t].y = p.svals[j0 + i];
      if (!fkm_in_range(e_[t].y, p.n, p.status)) e_[t].x = -1;   // the row is skipped
    }
  }
  int kedge = -1;   // lane 0: the key before the range; lane 1: the key after it
  if (lane == 0 && j0 > 0) kedge = p.skeys[j0 - 1];
  if (lane == 1 && j0 + nrows < p.n) kedge = p.skeys[j0 + nrows];
#pragma unroll
  for (int t = 0; t < SEG_RANGE / 32; ++t) {
    if (e_[t].x >= p.BK) e_[t].x = -1;   // rejected id: skip the row
    ws.kv[t * 32 + lane] = e_[t];
  }
  if (lane == 0) ws.kv[SEG_RANGE] = make_int2(-1, 0);
  const int key_before = __shfl_sync(0xffffffffu, kedge, 0);
  const int key_after = __shfl_sync(0xffffffffu, kedge, 1);
  __syncwarp();
  // run starts (ids that are rejected sort after every valid key, so the
  // valid rows are a prefix of the range)
  // With p.segstart, also the segment bounds: a run that starts (ends) in
  // this range starts (ends) its key's segment unless the key continues from
  // the range before (into the range after).
  int nruns = 0, nvalid = 0;
#pragma unroll
  for (int t = 0; t < SEG_RANGE / 32; ++t) {
    const int i = t * 32 + lane;
    const int k = ws.kv[i].x;
    const int kp = i > 0 ? ws.kv[i - 1].x : -1;
    const bool start = k >= 0 && (i == 0 || k != kp);
    const unsigned bal = __ballot_sync(0xffffffffu, start);
    if (start) ws.runs[nruns + __popc(bal & ((1u << lane) - 1u))] = (int16_t)i;
    nruns += __popc(bal);
    nvalid += __popc(__ballot_sync(0xffffffffu, k >= 0));
    if (p.segstart && k >= 0) {
      if (start && !(i == 0 && key_before == k)) p.segstart[k] = (int32_t)(j0 + i);
      const int kn = ws.kv[i + 1].x;   // the (-1, 0) entries past the range end it
      if (kn != k && !(i + 1 == nrows && key_after == k)) p.segend[k] = (int32_t)(j0 + i + 1);
    }
  }
  if (lane == 0) ws.runs[nruns] = (int16_t)nvalid;
  __syncwarp();

  const char* xb = static_cast<const char*>(p.x) + (int64_t)sub * 16;
  const int nsteps = (nrows + RPS - 1) / RPS;
  // Gather step s into ring slot s % SEG_STAGES.  Rows past the range read
  // the (-1, 0) entries (the staged tail and the sentinel), so the copy is a
  // zero fill from a valid address; so is the copy of a lane past the row's
  // last vector.  Each lane reads back only the piece it copied itself, so
  // the ring needs no warp barrier.
  const int novec = lane_has_vec ? 0 : (int)0x80000000;
  const int rb = (int)p.row_bytes;
  auto issue = [&](int s) {
    const int i = min(s * RPS + g, SEG_RANGE);
    const int2 e = ws.kv[i];
    cp_async_16(&ws.ring[s & (SEG_STAGES - 1)][lane], xb + (int64_t)e.y * rb, (e.x | novec) >= 0);
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < SEG_STAGES - 1; ++s) issue(s);

  // centroid rows for the objective: raw 16-byte piece of the next run's row
  uint4 chat_next = make_uint4(0, 0, 0, 0);
  // (batch, cluster) of a sorted key b*K + id: keys only grow along the
  // range, so the batch is found by division only when it changes
  int pf_b = -1, pf_base = 0;
  auto prefetch_chat = [&](int run) {
    if (!want_obj || run >= nruns || !lane_has_vec) return;
    const int kg = ws.kv[ws.runs[run]].x;
    if (pf_b < 0 || kg - pf_base >= p.oa.K) {
      pf_b = kg / p.oa.K;
      pf_base = pf_b * p.oa.K;
    }
    const int b = pf_b, k = kg - pf_base;
    const char* row = static_cast<const char*>(p.oa.chat) +
                      ((int64_t)b * p.oa.chat_bstride + (int64_t)k * p.Dfull) * elem_bytes_;
    chat_next = ldg_nc_v4(row + (int64_t)sub * 16);
  };
  prefetch_chat(0);

  // Lanes without a vector of the row (sub >= V) gather zeros and keep a zero
  // centroid piece, so they add nothing and need no test on the hot path.
  // fp64 sums live in shared memory (registers hold the fp32 partials)
  float2 acc2[E / 2], chat2[E / 2];
#pragma unroll
  for (int e = 0; e < E / 2; ++e) {
    acc2[e] = make_float2(0.0f, 0.0f);
    chat2[e] = make_float2(0.0f, 0.0f);
    ws.acc[e][lane] = make_double2(0.0, 0.0);
  }
  float2 obj2 = make_float2(0.0f, 0.0f);
  double obj = 0.0;
  int cur = -1, cur_b = -1, run = -1, run_start = 0, run_end = 0, since_fold = 0;
  const float2 neg1 = make_float2(-1.0f, -1.0f);
  auto fold_obj = [&]() {
    obj += (double)obj2.x + (double)obj2.y;
    obj2 = make_float2(0.0f, 0.0f);
  };
  // the fp32 partials hold at most 16 rows per lane before going to fp64
  auto fold = [&]() {
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      double2 a = ws.acc[e][lane];
      a.x += (double)acc2[e].x;
      a.y += (double)acc2[e].y;
      ws.acc[e][lane] = a;
      acc2[e] = make_float2(0.0f, 0.0f);
    }
    fold_obj();
    since_fold = 0;
  };
  // one row of the current run: this lane's vector of it
  auto add_row = [&](const uint4& v) {
    float2 f[E / 2];
    Vec<DT>::widen2(v, f);
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      acc2[e] = __fadd2_rn(acc2[e], f[e]);
      const float2 df = __ffma2_rn(chat2[e], neg1, f[e]);
      obj2 = __ffma2_rn(df, df, obj2);
    }
  };
  auto flush = [&](int end) {
    fold();
    const bool crossing = (run_start == 0 && key_before == cur) ||
                          (end == nrows && key_after == cur);
    double acc[E];
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      const double2 a = ws.acc[e][lane];
      acc[2 * e] = a.x;
      acc[2 * e + 1] = a.y;
      ws.acc[e][lane] = make_double2(0.0, 0.0);
    }
    flush_run<E, LPR>(p, cur, g, sub, lane_has_vec, !p.accumulate_all && !crossing,
                      end - run_start, acc);
  };
  // this lane's piece of the current batch's mean centroid (16-bit points),
  // loaded when the batch changes
  float2 m2[E / 2];
#pragma unroll
  for (int e = 0; e < E / 2; ++e) m2[e] = make_float2(0.0f, 0.0f);
  int cur_base = 0;   // cur_b * K
  auto start_run = [&](int kg, int i) {
    cur = kg;
    ++run;
    run_start = i;
    run_end = ws.runs[run + 1];
    if (!want_obj) return;
    fold_obj();
    if (cur_b < 0 || kg - cur_base >= p.oa.K) {   // a new batch (keys only grow)
      const int b = kg / p.oa.K;
      if (cur_b >= 0) {
        const double t = warp_sum(obj);
        if (lane == 0) atomicAdd(p.oa.obj + cur_b, t);
      }
      obj = 0.0;
      cur_b = b;
      cur_base = b * p.oa.K;
      if (p.oa.m && lane_has_vec) {
        const float2* mb =
            reinterpret_cast<const float2*>(p.oa.m + (int64_t)b * p.Dfull) + sub * (E / 2);
#pragma unroll
        for (int e = 0; e < E / 2; ++e) m2[e] = mb[e];
      }
    }
    if (lane_has_vec) {
      float2 c2[E / 2];
      Vec<DT>::widen2(chat_next, c2);
#pragma unroll
      for (int e = 0; e < E / 2; ++e) chat2[e] = __fadd2_rn(c2[e], m2[e]);
    }
    prefetch_chat(run + 1);
  };

  int s = 0;
#pragma unroll 1
  while (s < nsteps) {
    // a general step: the rows may start new runs
    issue(s + SEG_STAGES - 1);
    cp_async_wait_stages();   // step s has landed
    {
      const uint4 v = ws.ring[s & (SEG_STAGES - 1)][lane];
#pragma unroll
      for (int gg = 0; gg < RPS; ++gg) {
        const int i = s * RPS + gg;
        const int kg = ws.kv[i].x;   // same address in every lane: broadcast
        if (kg < 0) continue;
        if (kg != cur) {
          if (cur >= 0) flush(i);
          start_run(kg, i);
        }
        if (g == gg) add_row(v);
      }
    }
    if (++since_fold == 16) fold();
    ++s;
    // the steps that lie wholly inside the current run: keys sorted, so no
    // per-row test is needed
    const int s_end = cur >= 0 ? min(nsteps, run_end / RPS) : s;
#pragma unroll 1
    while (s < s_end) {
      issue(s + SEG_STAGES - 1);
      cp_async_wait_stages();
      add_row(ws.ring[s & (SEG_STAGES - 1)][lane]);
      if (++since_fold == 16) fold();
      ++s;
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  if (cur >= 0) flush(nvalid);
  if (want_obj && cur_b >= 0) {
    fold_obj();
    const double t = warp_sum(obj);
    if (lane == 0) atomicAdd(p.oa.obj + cur_b, t);
  }
}

// Direct objective of a given assignment, one warp per point row; grid.y = batch.
template <int DT>
__global__ void __launch_bounds__(256) objective_kernel(const void* __restrict__ x,
                                                        const int32_t* __restrict__ ids, int N,
                                                        int D, int V, int64_t row_bytes,
                                                        ObjArgs oa, int rows_per_block) {
  constexpr int E = Vec<DT>::E;
  __shared__ double red[8];
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = (int64_t)blockIdx.x * rows_per_block;
  double acc = 0.0;
  for (int64_t i = r0 + warp; i < r0 + rows_per_block && i < N; i += 8) {
    const int id = ids[(int64_t)b * N + i];
    if (id < 0 || id >= oa.K) continue;
    float d2 = 0.0f;
    for (int v = lane; v < V; v += 32) {   // the row's 16-byte vectors
      float f[E], c[E];
      Vec<DT>::widen(ldg_nc_v4(static_cast<const char*>(x) + ((int64_t)b * N + i) * row_bytes +
                               (int64_t)v * 16),
                     f);
      const char* crow = static_cast<const char*>(oa.chat) +
                         ((int64_t)b * oa.chat_bstride + (int64_t)id * D) * (row_bytes / D);
      Vec<DT>::widen(ldg_nc_v4(crow + (int64_t)v * 16), c);
      if (oa.m) {
        const float* mb = oa.m + (int64_t)b * D + (int64_t)v * E;
#pragma unroll
        for (int e = 0; e < E; ++e) c[e] += mb[e];
      }
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float df = f[e] - c[e];
        d2 = fmaf(df, df, d2);
      }
    }
    acc += (double)d2;
  }
  acc = warp_sum(acc);
  if (lane == 0) red[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += red[w];
    atomicAdd(oa.obj + b, t);
  }
}

struct FinParams {
  int B, K, D;
  const int32_t* segstart;
  const int32_t* segend;
  double* sums64;
  const float* prev;
  float* centers;
  int32_t* counts;
  double* shiftk;
  const int32_t* counts_in;  // out-of-core: accumulated counts (segstart/end unused)
  const double* counts_in64;  // shard partials reduced across GPUs: counts as fp64
  int range;                 // the segment sums' rows per warp range
  bool clear_sums;           // zero sums64 after use (the library's own accumulators)
};

// One warp per cluster.  When D is a multiple of 4 each lane moves four
// consecutive elements per step (16-byte loads and stores), so a cluster of
// D <= 128 takes one step.
__global__ void finalize_kernel(FinParams p) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  const int64_t key = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (key >= (int64_t)p.B * p.K) return;
  int32_t nk;
  bool interior = false;
  if (p.counts_in64) {
    nk = (int32_t)p.counts_in64[key];
  } else if (p.counts_in) {
    nk = p.counts_in[key];
  } else {
    const int32_t s = p.segstart[key], t = p.segend[key];
    nk = t - s;
    interior = nk > 0 && (s / p.range) == ((t - 1) / p.range);
  }
  if (lane == 0 && p.counts) p.counts[key] = nk;
  double sh = 0.0;
  if ((p.D & 3) == 0) {
    for (int d = 4 * lane; d < p.D; d += 128) {
      const int64_t e = key * p.D + d;
      const float4 pv = *reinterpret_cast<const float4*>(p.prev + e);
      float4 v;
      if (nk == 0) {
        v = pv;
      } else if (interior) {
        v = *reinterpret_cast<const float4*>(p.centers + e);
      } else {
        double2* s2 = reinterpret_cast<double2*>(p.sums64 + e);
        const double2 a = s2[0], b = s2[1];
        const double n = (double)nk;
        v = make_float4((float)(a.x / n), (float)(a.y / n), (float)(b.x / n), (float)(b.y / n));
        if (p.clear_sums) {   // leave the accumulator clean for the next update
          s2[0] = make_double2(0.0, 0.0);
          s2[1] = make_double2(0.0, 0.0);
        }
      }
      *reinterpret_cast<float4*>(p.centers + e) = v;
      const double d0 = (double)v.x - (double)pv.x, d1 = (double)v.y - (double)pv.y;
      const double d2 = (double)v.z - (double)pv.z, d3 = (double)v.w - (double)pv.w;
      sh += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
    }
  } else {
    for (int d = lane; d < p.D; d += 32) {
      const int64_t e = key * p.D + d;
      const float prev = p.prev[e];
      float v;
      if (nk == 0) {
        v = prev;
      } else if (interior) {
        v = p.centers[e];
      } else {
        v = (float)(p.sums64[e] / (double)nk);
        if (p.clear_sums) p.sums64[e] = 0.0;
      }
      p.centers[e] = v;
      const double df = (double)v - (double)prev;
      sh += df * df;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sh += __shfl_xor_sync(0xffffffffu, sh, o);
  if (lane == 0) p.shiftk[key] = sh;
}

// Finalize for dot-product and cosine k-means (one warp per cluster).  The
// new centroid is the mean of the cluster's points (dot), or its direction
// scaled to unit length (cosine: the mean's direction is the sum's); an empty
// cluster, or a cosine cluster whose sum is zero, keeps prev.  objk[key] is
// the cluster's share of the objective of the assignment just summed,
// s_k . c~ with c~ = prev (dot) or prev / ||prev|| (cosine), s_k the sum of
// its points: the fp64 sums of a crossing run, or n times the mean the
// segment sums wrote for an interior one.
struct FinSimParams {
  int B, K, D, metric, range;
  const int32_t* segstart;
  const int32_t* segend;
  const int32_t* counts_in;  // out-of-core: accumulated counts, every sum in sums64
  double* sums64;
  const float* prev;
  float* centers;
  int32_t* counts;
  double* shiftk;
  double* objk;
  bool clear_sums;
};

__global__ void finalize_sim_kernel(FinSimParams p) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  const int64_t key = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (key >= (int64_t)p.B * p.K) return;
  int32_t nk;
  bool interior = false;
  if (p.counts_in) {
    nk = p.counts_in[key];
  } else {
    const int32_t s0 = p.segstart[key], t0 = p.segend[key];
    nk = t0 - s0;
    interior = nk > 0 && (s0 / p.range) == ((t0 - 1) / p.range);
  }
  const bool cosine = p.metric == FKM_METRIC_COSINE;
  const double n = (double)nk;
  if (p.D <= 128 && (p.D & 3) == 0) {
    // one 16-byte piece per lane holds the whole cluster: one pass of loads
    const int d = 4 * lane;
    const bool on = d < p.D;
    const int64_t e = key * p.D + d;
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
        const double2 a = s2[0], b = s2[1];
        sd[0] = a.x;
        sd[1] = a.y;
        sd[2] = b.x;
        sd[3] = b.y;
        v = make_float4((float)(a.x / n), (float)(a.y / n), (float)(b.x / n), (float)(b.y / n));
        if (p.clear_sums) {
          s2[0] = make_double2(0.0, 0.0);
          s2[1] = make_double2(0.0, 0.0);
        }
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
    if (lane == 0) {
      p.shiftk[key] = sh;
      p.objk[key] = cosine ? (pn > 0.0 ? sp / pn : 0.0) : sp;
      if (p.counts) p.counts[key] = nk;
    }
    return;
  }
  // pass 1: ||mean||^2, ||prev||^2 and sum . prev
  double vv = 0.0, pp = 0.0, sp = 0.0;
  for (int d = lane; d < p.D; d += 32) {
    const int64_t e = key * p.D + d;
    const double pv = (double)p.prev[e];
    pp += pv * pv;
    if (nk > 0) {
      double sd;
      float v;
      if (interior) {
        v = p.centers[e];
        sd = (double)v * n;
      } else {
        sd = p.sums64[e];
        v = (float)(sd / n);
      }
      vv += (double)v * (double)v;
      sp += sd * pv;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vv += __shfl_xor_sync(0xffffffffu, vv, o);
    pp += __shfl_xor_sync(0xffffffffu, pp, o);
    sp += __shfl_xor_sync(0xffffffffu, sp, o);
  }
  const double pn = sqrt(pp), vn = sqrt(vv);
  const double obj = cosine ? (pn > 0.0 ? sp / pn : 0.0) : sp;
  const bool keep = nk == 0 || (cosine && !(vv > 0.0));
  // pass 2: the new centroid and its shift
  double sh = 0.0;
  for (int d = lane; d < p.D; d += 32) {
    const int64_t e = key * p.D + d;
    const float pv = p.prev[e];
    float out = pv;
    if (!keep) {
      const float v = interior ? p.centers[e] : (float)(p.sums64[e] / n);
      out = cosine ? (float)((double)v / vn) : v;
    }
    if (nk > 0 && !interior && p.clear_sums) p.sums64[e] = 0.0;
    p.centers[e] = out;
    const double df = (double)out - (double)pv;
    sh += df * df;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sh += __shfl_xor_sync(0xffffffffu, sh, o);
  if (lane == 0) {
    p.shiftk[key] = sh;
    p.objk[key] = obj;
    if (p.counts) p.counts[key] = nk;
  }
}

// one block per batch; fixed-order tree sum
__global__ void __launch_bounds__(256) batch_reduce_kernel(int K, const double* __restrict__ shiftk,
                                                           double* shift_out, double* max_shift) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  __shared__ double s1[256];
  const int b = blockIdx.x;
  double a = 0.0;
  for (int k = threadIdx.x; k < K; k += 256) a += shiftk[(int64_t)b * K + k];
  s1[threadIdx.x] = a;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) s1[threadIdx.x] += s1[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (shift_out) shift_out[b] = s1[0];
    if (max_shift)  // shift >= 0: the bit pattern orders like the value
      atomicMax(reinterpret_cast<unsigned long long*>(max_shift),
                (unsigned long long)__double_as_longlong(s1[0]));
  }
}

template <int DT, int RPS>
fkm_status run_segsum(const SegParams& sp, cudaStream_t st) {
  const int64_t nranges = ceil_div(sp.n, sp.range);
  const int64_t blocks = ceil_div(nranges, SEG_WARPS);
  FKM_CUDA_TRY(launch_pdl((segsum_kernel<DT, RPS>), dim3((unsigned)blocks), dim3(SEG_WARPS * 32),
                          SEG_SMEM_BYTES, st, sp));
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

template <int DT>
fkm_status set_segsum_smem() {
  const int b = (int)SEG_SMEM_BYTES;
  FKM_CUDA_TRY(cudaFuncSetAttribute(segsum_kernel<DT, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, b));
  FKM_CUDA_TRY(cudaFuncSetAttribute(segsum_kernel<DT, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, b));
  FKM_CUDA_TRY(cudaFuncSetAttribute(segsum_kernel<DT, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, b));
  FKM_CUDA_TRY(cudaFuncSetAttribute(segsum_kernel<DT, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, b));
  FKM_CUDA_TRY(cudaFuncSetAttribute(segsum_kernel<DT, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, b));
  FKM_CUDA_TRY(cudaFuncSetAttribute(segsum_kernel<DT, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, b));
  return FKM_OK;
}

template <int DT>
fkm_status run_segsum_dt(const SegParams& sp, cudaStream_t st) {
  int lpr = 1;
  while (lpr < sp.V) lpr <<= 1;
  switch (32 / lpr) {
    case 1: return run_segsum<DT, 1>(sp, st);
    case 2: return run_segsum<DT, 2>(sp, st);
    case 4: return run_segsum<DT, 4>(sp, st);
    case 8: return run_segsum<DT, 8>(sp, st);
    case 16: return run_segsum<DT, 16>(sp, st);
    default: return run_segsum<DT, 32>(sp, st);
  }
}

}  // namespace

int segsum_range_rows(int64_t n) {
  // about two rounds of the warps that fit on the GPU at once
  const int64_t warps = (int64_t)num_sms() * SEG_WARPS * FKM_SEG_MIN_BLOCKS * 2;
  int64_t r = round_up(ceil_div(n, warps), 32);
  if (r < 32) r = 32;
  if (r > SEG_RANGE) r = SEG_RANGE;
  return (int)r;
}

fkm_status segsum_prepare() {
  static bool done[64] = {false};
  int dev = 0;
  FKM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && done[dev]) return FKM_OK;
  FKM_TRY(set_segsum_smem<FKM_BF16>());
  FKM_TRY(set_segsum_smem<FKM_F16>());
  FKM_TRY(set_segsum_smem<FKM_F32>());
  if (dev >= 0 && dev < 64) done[dev] = true;
  return FKM_OK;
}

fkm_status clear_seg_bounds(int BK, int32_t* segstart, int32_t* segend, cudaStream_t st) {
  FKM_CUDA_TRY(cudaMemsetAsync(segstart, 0, sizeof(int32_t) * (size_t)BK, st));
  FKM_CUDA_TRY(cudaMemsetAsync(segend, 0, sizeof(int32_t) * (size_t)BK, st));
  return FKM_OK;
}

fkm_status launch_segsum(const void* x, int dtype, int D, const int32_t* skeys,
                         const int32_t* svals, int64_t n, int BK, double* sums64, float* centers,
                         bool accumulate_all, const ObjArgs& oa, cudaStream_t st, int range,
                         unsigned long long* atomics, int32_t* segstart, int32_t* segend,
                         int* status) {
  if (n == 0) return FKM_OK;
  if (range <= 0) range = segsum_range_rows(n);
  FKM_TRY(segsum_prepare());
  const int eb = elem_bytes(dtype);
  const int slab = 512 / eb;   // columns per launch: 512-byte row pieces
  for (int c0 = 0; c0 < D; c0 += slab) {
    SegParams sp;
    sp.x = static_cast<const char*>(x) + (int64_t)c0 * eb;
    sp.skeys = skeys;
    sp.svals = svals;
    sp.n = n;
    sp.D = D - c0 < slab ? D - c0 : slab;
    sp.Dfull = D;
    sp.BK = BK;
    sp.row_bytes = (int64_t)D * eb;
    sp.ebytes = eb;
    sp.V = (int)((int64_t)sp.D * eb / 16);
    sp.range = range;
    sp.sums64 = sums64 + c0;
    sp.centers = centers ? centers + c0 : nullptr;
    sp.accumulate_all = accumulate_all;
    sp.oa = oa;
    sp.atomics = atomics;
    sp.segstart = c0 == 0 ? segstart : nullptr;   // the first column slab writes them
    sp.segend = c0 == 0 ? segend : nullptr;
    sp.status = status;
    if (oa.chat) sp.oa.chat = static_cast<const char*>(oa.chat) + (int64_t)c0 * eb;
    if (oa.m) sp.oa.m = oa.m + c0;
    if (dtype == FKM_BF16) FKM_TRY(run_segsum_dt<FKM_BF16>(sp, st));
    else if (dtype == FKM_F16) FKM_TRY(run_segsum_dt<FKM_F16>(sp, st));
    else FKM_TRY(run_segsum_dt<FKM_F32>(sp, st));
  }
  return FKM_OK;
}

fkm_status launch_objective(const void* x, int dtype, int B, int N, int D, const int32_t* ids,
                            const ObjArgs& oa, cudaStream_t st) {
  const int64_t row_bytes = (int64_t)D * elem_bytes(dtype);
  const int V = (int)(row_bytes / 16);
  const int rpb = 64;
  dim3 grid((unsigned)ceil_div(N, rpb), (unsigned)B);
  if (dtype == FKM_BF16)
    objective_kernel<FKM_BF16><<<grid, 256, 0, st>>>(x, ids, N, D, V, row_bytes, oa, rpb);
  else if (dtype == FKM_F16)
    objective_kernel<FKM_F16><<<grid, 256, 0, st>>>(x, ids, N, D, V, row_bytes, oa, rpb);
  else
    objective_kernel<FKM_F32><<<grid, 256, 0, st>>>(x, ids, N, D, V, row_bytes, oa, rpb);
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

fkm_status launch_finalize(int B, int K, int D, const int32_t* segstart, const int32_t* segend,
                           const int32_t* counts_in, double* sums64, const float* prev,
                           float* centers, int32_t* counts, double* shiftk, cudaStream_t st,
                           int range, bool clear_sums, const double* counts_in64) {
  FinParams fp;
  fp.counts_in64 = counts_in64;
  fp.range = range;
  fp.clear_sums = clear_sums;
  fp.B = B;
  fp.K = K;
  fp.D = D;
  fp.segstart = segstart;
  fp.segend = segend;
  fp.sums64 = sums64;
  fp.prev = prev;
  fp.centers = centers;
  fp.counts = counts;
  fp.shiftk = shiftk;
  fp.counts_in = counts_in;
  const int64_t keys = (int64_t)B * K;
  const int wpb = 8;
  FKM_CUDA_TRY(launch_pdl(finalize_kernel, dim3((unsigned)ceil_div(keys, wpb)), dim3(wpb * 32), 0,
                          st, fp));
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

fkm_status launch_finalize_sim(int B, int K, int D, int metric, const int32_t* segstart,
                               const int32_t* segend, double* sums64, const float* prev,
                               float* centers, int32_t* counts, double* shiftk, double* objk,
                               cudaStream_t st, int range, const int32_t* counts_in) {
  FinSimParams fp;
  fp.counts_in = counts_in;
  fp.B = B;
  fp.K = K;
  fp.D = D;
  fp.metric = metric;
  fp.range = range;
  fp.segstart = segstart;
  fp.segend = segend;
  fp.sums64 = sums64;
  fp.prev = prev;
  fp.centers = centers;
  fp.counts = counts;
  fp.shiftk = shiftk;
  fp.objk = objk;
  fp.clear_sums = true;
  const int64_t keys = (int64_t)B * K;
  FKM_CUDA_TRY(launch_pdl(finalize_sim_kernel, dim3((unsigned)ceil_div(keys, 8)), dim3(256), 0, st,
                          fp));
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

fkm_status launch_batch_reduce(int B, int K, const double* shiftk, double* shift_out,
                               double* max_shift, cudaStream_t st) {
  FKM_CUDA_TRY(launch_pdl(batch_reduce_kernel, dim3(B), dim3(256), 0, st,
                          K, shiftk, shift_out, max_shift));
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

}  // namespace fkm
