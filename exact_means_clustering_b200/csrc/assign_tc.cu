// FlashAssign on sm_100a: nearest-centroid search without a distance matrix.
//
// "Flash-KMeans: Fast and Memory-Efficient Exact K-Means" summary, section
// "Method" (FlashAssign), and the "Flash-KMeans：快速且内存高效精确K-Means聚类"
// summary, section 方法步骤详情 step (1): tile the points (B_N) and the
// centroids (B_K); per point keep a running (min score, index) that starts at
// +inf; per centroid tile compute the local B_N x B_K block on chip, take its
// row minima and fold them into the running state; write the final index once.
// The score is ||c||^2 - 2 x.c (the same page, section 核心方法: ||x||^2 is
// constant per point and does not change the argmin).
//
// B200 design (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: the point tile [128 x D] once per work item into
//               one of nA buffers, centroid tiles [256 x 64] through an
//               nS-stage ring (128-byte swizzle, no multicast).
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators)
//               and issues tcgen05.mma (M=128, N=256, K=16) from one thread.
//   warps 2-9   epilogue, two warpgroups: TMEM lane t = point t of the tile;
//               warpgroup h reads columns [128h, 128h + 128) of every
//               accumulator (tcgen05.ld), forms score = ||q(c)||^2 - 2 acc with
//               packed fp32x2 FMAs and keeps its running minimum with 3-input
//               min trees; the two halves are merged per work item.  Ties go
//               to the lowest centroid index.
// Accumulator double buffering lets the MMAs of tile t+1 run while the
// epilogue reduces tile t; A double buffering overlaps the next work item's
// point load with the current one's MMAs.
//
// fp32 points: x = xh + xl and c = ch + cl with bf16 parts; three MMAs per
// K-chunk (xh.ch + xh.cl + xl.ch) give the product to ~2^-17 relative
// (split-bf16 products, Henry, Tang and Heinecke, ARITH 2019).
//
// Every mbarrier wait is bounded (globaltimer); when one runs out the CTA sets
// ST_TIMEOUT in the status word, every role leaves its loop, in-flight copies
// and MMAs are drained with bounded waits and TMEM is released.  The epilogue
// synchronises only through mbarriers (no named barriers), so a role that
// leaves early cannot strand the others.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cfloat>
#include <cstddef>
#include <cstdio>

#include "fkm_internal.cuh"
#include "ptx_sm100.cuh"

namespace fkm {
namespace {

constexpr uint64_t kWaitTimeoutNs = 4000000000ull;  // 4 s

struct AssignKParams {
  int B, N, Kp;
  int nD;          // 64-wide D chunks
  int m_tiles;     // point tiles per batch
  int k_tiles;     // centroid tiles per batch
  int n_work;      // B * m_tiles
  int nA, nS;      // point buffers, centroid stages
  uint32_t a_bytes, s_bytes;
  uint32_t idesc;
  const float* cn;
  const float* xn;  // ||x||^2, comparison mode only
  int32_t* ids;
  int* status;
  int K;           // real centroids (materialised rows are K wide)
  float* dist;     // comparison mode only: the full [B, N, K] distance matrix
};

struct __align__(8) SmemCtl {
  uint64_t a_full[2], a_empty[2];
  uint64_t b_full[8], b_empty[8];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t cn_full[2];
  uint64_t merge_full, merge_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  __align__(16) float cn_s[2][BN];   // read with 16-byte loads
  float2 merge[BM];   // (best score, index as float bits) of warpgroup 1
};
static_assert(offsetof(SmemCtl, cn_s) % 16 == 0, "cn_s must be 16-byte aligned");

// Per epilogue thread, the scores of the chunk that last improved its
// running minimum (32 floats), with the 16-byte units rotated by lane so the
// predicated stores of a warp hit distinct banks.
constexpr int kSaveBytes = 256 * 32 * 4;

__device__ __forceinline__ float2 u2f2(uint32_t a, uint32_t b) {
  return make_float2(__uint_as_float(a), __uint_as_float(b));
}

// Minimum of 32 scores with 3-input min instructions.
__device__ __forceinline__ float min32(const float (&s)[32]) {
  float m0 = ptx::fmin3(s[0], s[1], s[2]);
  float m1 = ptx::fmin3(s[3], s[4], s[5]);
  float m2 = ptx::fmin3(s[6], s[7], s[8]);
  float m3 = ptx::fmin3(s[9], s[10], s[11]);
  float m4 = ptx::fmin3(s[12], s[13], s[14]);
  float m5 = ptx::fmin3(s[15], s[16], s[17]);
  float m6 = ptx::fmin3(s[18], s[19], s[20]);
  float m7 = ptx::fmin3(s[21], s[22], s[23]);
  float m8 = ptx::fmin3(s[24], s[25], s[26]);
  float m9 = ptx::fmin3(s[27], s[28], s[29]);
  float m10 = fminf(s[30], s[31]);
  float n0 = ptx::fmin3(m0, m1, m2);
  float n1 = ptx::fmin3(m3, m4, m5);
  float n2 = ptx::fmin3(m6, m7, m8);
  float n3 = fminf(m9, m10);
  return fminf(ptx::fmin3(n0, n1, n2), n3);
}

// Scores of one 32-column chunk, s = cn - 2 acc, folded into (best, bcol).
// A chunk replaces the running minimum only when strictly smaller; then its
// scores are saved so the lowest column holding the minimum can be found once
// per work item (find_first), which keeps the lowest centroid index among
// exact ties without a per-chunk search.
__device__ __forceinline__ void fold_chunk(const uint32_t (&r)[32], const float* cn, int col0,
                                           float& best, int& bcol, float4* save, int rot) {
  float s[32];
  const float2 m2 = make_float2(-2.0f, -2.0f);
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 c4 = *reinterpret_cast<const float4*>(cn + j);
    const float2 v0 = __ffma2_rn(u2f2(r[j], r[j + 1]), m2, make_float2(c4.x, c4.y));
    const float2 v1 = __ffma2_rn(u2f2(r[j + 2], r[j + 3]), m2, make_float2(c4.z, c4.w));
    s[j] = v0.x;
    s[j + 1] = v0.y;
    s[j + 2] = v1.x;
    s[j + 3] = v1.y;
  }
  const float cm = min32(s);
  if (cm < best) {
    best = cm;
    bcol = col0;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      save[k ^ rot] = make_float4(s[4 * k], s[4 * k + 1], s[4 * k + 2], s[4 * k + 3]);
  }
}

// Lowest position j in the saved chunk whose score equals best.
__device__ __forceinline__ int find_first(const float4* save, int rot, float best) {
  uint32_t mask = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float4 v = save[k ^ rot];
    mask |= (uint32_t)(v.x == best) << (4 * k);
    mask |= (uint32_t)(v.y == best) << (4 * k + 1);
    mask |= (uint32_t)(v.z == best) << (4 * k + 2);
    mask |= (uint32_t)(v.w == best) << (4 * k + 3);
  }
  return mask ? __ffs(mask) - 1 : 0;
}

// kDist = true is the comparison ("standard") mode: the same tensor-core tiles,
// but the epilogue writes every distance ||x - c_hat||^2 = ||x - m||^2 +
// norm_k - 2 x.q(c_k - m) to HBM instead of reducing it, as the pages'
// baseline assignment does.
template <bool kSplit, bool kDist>
__global__ void __launch_bounds__(ASSIGN_THREADS, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tm_x,   // points (hi part when split)
                     const __grid_constant__ CUtensorMap tm_xl,  // lo part (split only)
                     const __grid_constant__ CUtensorMap tm_c,   // centroids (hi part when split)
                     const __grid_constant__ CUtensorMap tm_cl,  // lo part (split only)
                     const AssignKParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* a_base = smem;
  uint8_t* b_base = a_base + (size_t)p.nA * p.a_bytes;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(b_base + (size_t)p.nS * p.s_bytes);
  float4* save_base = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(ctl) +
                                                ((sizeof(SmemCtl) + 127) & ~size_t(127)));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &ctl->abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.nA; ++i) {
      ptx::mbar_init(&ctl->a_full[i], 1);
      ptx::mbar_init(&ctl->a_empty[i], 1);
    }
    for (int i = 0; i < p.nS; ++i) {
      ptx::mbar_init(&ctl->b_full[i], 1);
      ptx::mbar_init(&ctl->b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&ctl->acc_full[i], 1);
      ptx::mbar_init(&ctl->acc_empty[i], 8);
      ptx::mbar_init(&ctl->cn_full[i], 256);
    }
    ptx::mbar_init(&ctl->merge_full, 128);
    ptx::mbar_init(&ctl->merge_empty, 128);
    ptx::mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&ctl->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_x);
      ptx::prefetch_tmap(&tm_c);
      if (kSplit) {
        ptx::prefetch_tmap(&tm_xl);
        ptx::prefetch_tmap(&tm_cl);
      }
      uint32_t a_arms = 0, s_arms = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.n_work && ok; w += gridDim.x) {
        const int b = w / p.m_tiles, mt = w % p.m_tiles;
        const int ab = a_arms % p.nA;
        const uint32_t apar = ((a_arms / p.nA) & 1) ^ 1;
        if (!ptx::mbar_wait_bounded(&ctl->a_empty[ab], apar, abort_flag, p.status, ST_TIMEOUT,
                                    kWaitTimeoutNs)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&ctl->a_full[ab], p.a_bytes);
        uint8_t* abuf = a_base + (size_t)ab * p.a_bytes;
        for (int dc = 0; dc < p.nD; ++dc) {
          ptx::tma_load_3d(abuf + dc * A_CHUNK_BYTES, &tm_x, &ctl->a_full[ab], dc * KC, mt * BM, b);
          if (kSplit)
            ptx::tma_load_3d(abuf + (p.nD + dc) * A_CHUNK_BYTES, &tm_xl, &ctl->a_full[ab], dc * KC,
                             mt * BM, b);
        }
        ++a_arms;
        for (int kt = 0; kt < p.k_tiles && ok; ++kt) {
          // one stage per 64-wide chunk; split operands put hi and lo in
          // consecutive stages
          for (int q = 0; q < p.nD * (kSplit ? 2 : 1); ++q) {
            const int dc = kSplit ? (q >> 1) : q;
            const int sb = s_arms % p.nS;
            const uint32_t spar = ((s_arms / p.nS) & 1) ^ 1;
            if (!ptx::mbar_wait_bounded(&ctl->b_empty[sb], spar, abort_flag, p.status, ST_TIMEOUT,
                                        kWaitTimeoutNs)) { ok = false; break; }
            ptx::mbar_arrive_expect_tx(&ctl->b_full[sb], p.s_bytes);
            uint8_t* sbuf = b_base + (size_t)sb * p.s_bytes;
            ptx::tma_load_3d(sbuf, (kSplit && (q & 1)) ? &tm_cl : &tm_c, &ctl->b_full[sb],
                             dc * KC, kt * BN, b);
            ++s_arms;
          }
        }
      }
      // Drain: every buffer's most recent load must have landed before exit.
      for (uint32_t i = 0; i < (uint32_t)p.nA && i < a_arms; ++i) {
        uint32_t last = i + p.nA * ((a_arms - 1 - i) / p.nA);
        ptx::mbar_wait_bounded(&ctl->a_full[i], (last / p.nA) & 1, abort_flag, p.status,
                               ST_TIMEOUT, kWaitTimeoutNs);
      }
      for (uint32_t i = 0; i < (uint32_t)p.nS && i < s_arms; ++i) {
        uint32_t last = i + p.nS * ((s_arms - 1 - i) / p.nS);
        ptx::mbar_wait_bounded(&ctl->b_full[i], (last / p.nS) & 1, abort_flag, p.status,
                               ST_TIMEOUT, kWaitTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t a_uses = 0, s_uses = 0, acc_uses = 0;
      bool ok = true;
      bool issued = false;
      for (int w = blockIdx.x; w < p.n_work && ok; w += gridDim.x) {
        const int ab = a_uses % p.nA;
        if (!ptx::mbar_wait_bounded(&ctl->a_full[ab], (a_uses / p.nA) & 1, abort_flag, p.status,
                                    ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t a_addr = ptx::smem_u32(a_base + (size_t)ab * p.a_bytes);
        for (int kt = 0; kt < p.k_tiles && ok; ++kt) {
          const int acc = acc_uses & 1;
          if (!ptx::mbar_wait_bounded(&ctl->acc_empty[acc], ((acc_uses >> 1) & 1) ^ 1, abort_flag,
                                      p.status, ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          for (int q = 0; q < p.nD * (kSplit ? 2 : 1); ++q) {
            const int dc = kSplit ? (q >> 1) : q;
            const int sb = s_uses % p.nS;
            if (!ptx::mbar_wait_bounded(&ctl->b_full[sb], (s_uses / p.nS) & 1, abort_flag,
                                        p.status, ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t b_addr = ptx::smem_u32(b_base + (size_t)sb * p.s_bytes);
            const uint32_t xa = a_addr + dc * A_CHUNK_BYTES;
            if (!(kSplit && (q & 1))) {
              // xh . ch (or x . q(c)); the first product of the tile overwrites
#pragma unroll
              for (int k = 0; k < KC / 16; ++k)
                ptx::mma_f16_ss(d_tmem, ptx::umma_desc_sw128(xa + 32 * k),
                                ptx::umma_desc_sw128(b_addr + 32 * k), p.idesc,
                                (q > 0 || k > 0) ? 1u : 0u);
              if (kSplit) {   // xl . ch
                const uint32_t xl = a_addr + (p.nD + dc) * A_CHUNK_BYTES;
#pragma unroll
                for (int k = 0; k < KC / 16; ++k)
                  ptx::mma_f16_ss(d_tmem, ptx::umma_desc_sw128(xl + 32 * k),
                                  ptx::umma_desc_sw128(b_addr + 32 * k), p.idesc, 1u);
              }
            } else {          // xh . cl
#pragma unroll
              for (int k = 0; k < KC / 16; ++k)
                ptx::mma_f16_ss(d_tmem, ptx::umma_desc_sw128(xa + 32 * k),
                                ptx::umma_desc_sw128(b_addr + 32 * k), p.idesc, 1u);
            }
            issued = true;
            ptx::mma_commit(&ctl->b_empty[sb]);
            ++s_uses;
          }
          if (!ok) break;
          ptx::mma_commit(&ctl->acc_full[acc]);
          ++acc_uses;
        }
        if (!ok) break;
        ptx::mma_commit(&ctl->a_empty[ab]);
        ++a_uses;
      }
      // Drain: all MMAs this thread issued must finish before TMEM is freed.
      if (issued) {
        ptx::mma_commit(&ctl->drain);
        ptx::mbar_wait_bounded(&ctl->drain, 0, abort_flag, p.status, ST_TIMEOUT, kWaitTimeoutNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;          // 0..255
    const int ew = warp - 2;                  // epilogue warp 0..7
    const int half = ew >> 2;                 // columns [128*half, 128*half + 128) of a tile
    const int quad = warp & 3;                // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;         // point within the tile
    const int rot = lane & 7;
    float4* save = save_base + (size_t)(ew * 32 + lane) * 8;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    uint32_t acc_uses = 0, items = 0;
    bool ok = true;
    // ||q(c)||^2 of the next tile, loaded one tile ahead so the global load
    // is off the critical path
    float cn_pre = (blockIdx.x < (unsigned)p.n_work)
                       ? p.cn[(size_t)(blockIdx.x / p.m_tiles) * p.Kp + et] : 0.0f;
    for (int w = blockIdx.x; w < p.n_work && ok; w += gridDim.x, ++items) {
      const int b = w / p.m_tiles, mt = w % p.m_tiles;
      float best = INFINITY;
      int bcol = 0;
      for (int kt = 0; kt < p.k_tiles; ++kt) {
        const int acc = acc_uses & 1;
        const uint32_t par = (acc_uses >> 1) & 1;
        const float cn_cur = cn_pre;
        if (kt + 1 < p.k_tiles)
          cn_pre = p.cn[(size_t)b * p.Kp + (size_t)(kt + 1) * BN + et];
        else if (w + (int)gridDim.x < p.n_work)
          cn_pre = p.cn[(size_t)((w + gridDim.x) / p.m_tiles) * p.Kp + et];
        // Stage ||q(c)||^2 of this centroid tile in shared memory.  Buffer acc
        // was last read two tiles ago, and every thread finished that tile
        // before it arrived for the previous one, so it is free to overwrite.
        ctl->cn_s[acc][et] = cn_cur;
        ptx::mbar_arrive(&ctl->cn_full[acc]);
        if (!ptx::mbar_wait_bounded(&ctl->cn_full[acc], par, abort_flag, p.status, ST_TIMEOUT,
                                    kWaitTimeoutNs)) { ok = false; break; }
        if (!ptx::mbar_wait_bounded(&ctl->acc_full[acc], par, abort_flag, p.status, ST_TIMEOUT,
                                    kWaitTimeoutNs)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t taddr = lane_addr + (uint32_t)(acc * BN + half * 128);
        const float* cn_s = ctl->cn_s[acc] + half * 128;
        const int colb = kt * BN + half * 128;
        uint32_t r0[32], r1[32];
        if (kDist) {
          const int gi = mt * BM + row;
          const float xv = (gi < p.N) ? p.xn[(size_t)b * p.N + gi] : 0.0f;
          float* drow = p.dist + ((size_t)b * p.N + (gi < p.N ? gi : 0)) * p.K;
          const bool vec4 = (p.K & 3) == 0;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            ptx::tmem_ld32(taddr + c * 32, r0);
            ptx::tmem_wait_ld32(r0);
            if (c == 3) {
              ptx::tc_fence_before();
              __syncwarp();
              if (lane == 0) ptx::mbar_arrive(&ctl->acc_empty[acc]);
            }
            const int col0 = colb + c * 32;
            if (gi < p.N && col0 < p.K) {
              float dv[32];
#pragma unroll
              for (int j = 0; j < 32; ++j)
                dv[j] = xv + fmaf(-2.0f, __uint_as_float(r0[j]), cn_s[c * 32 + j]);
              if (vec4 && col0 + 32 <= p.K) {
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                  *reinterpret_cast<float4*>(drow + col0 + j) =
                      make_float4(dv[j], dv[j + 1], dv[j + 2], dv[j + 3]);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (col0 + j < p.K) drow[col0 + j] = dv[j];
              }
            }
          }
          ++acc_uses;
          continue;
        }
        // all 128 of this warp's columns in flight at once, one wait, then the
        // accumulator goes straight back to the MMA warp
        uint32_t r2[32], r3[32];
        ptx::tmem_ld32(taddr, r0);
        ptx::tmem_ld32(taddr + 32, r1);
        ptx::tmem_ld32(taddr + 64, r2);
        ptx::tmem_ld32(taddr + 96, r3);
        ptx::tmem_wait_ld128(r0, r1, r2, r3);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctl->acc_empty[acc]);
        fold_chunk(r0, cn_s, colb, best, bcol, save, rot);
        fold_chunk(r1, cn_s + 32, colb + 32, best, bcol, save, rot);
        fold_chunk(r2, cn_s + 64, colb + 64, best, bcol, save, rot);
        fold_chunk(r3, cn_s + 96, colb + 96, best, bcol, save, rot);
        ++acc_uses;
      }
      if (!ok) break;
      if (kDist) continue;
      const int idx = bcol + find_first(save, rot, best);
      // merge the two column halves of each row
      const uint32_t mpar = items & 1;
      if (half == 1) {
        if (!ptx::mbar_wait_bounded(&ctl->merge_empty, mpar ^ 1, abort_flag, p.status,
                                    ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
        ctl->merge[row] = make_float2(best, __int_as_float(idx));
        ptx::mbar_arrive(&ctl->merge_full);
      } else {
        if (!ptx::mbar_wait_bounded(&ctl->merge_full, mpar, abort_flag, p.status, ST_TIMEOUT,
                                    kWaitTimeoutNs)) { ok = false; break; }
        const float2 o = ctl->merge[row];
        ptx::mbar_arrive(&ctl->merge_empty);
        const int oidx = __float_as_int(o.y);
        const int fidx = (o.x < best || (o.x == best && oidx < idx)) ? oidx : idx;
        const int gi = mt * BM + row;
        if (gi < p.N) p.ids[(size_t)b * p.N + gi] = fidx;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D map over [batches][rows][cols] 16-bit elements with a row pitch of
// row_elems; the box is box_cols x box_rows x 1 with the 128-byte swizzle.
// Elements outside [cols) x [rows) read as zero.
fkm_status make_map(CUtensorMap* m, const void* base, bool bf16, int cols, int rows, int batches,
                    int row_elems, int box_cols, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    set_error("cuTensorMapEncodeTiled is not available from the CUDA driver");
    return FKM_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batches};
  cuuint64_t strides[2] = {(cuuint64_t)row_elems * 2, (cuuint64_t)row_elems * 2 * rows};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (%d) for a %d x %d x %d map", (int)r, cols, rows,
              batches);
    return FKM_ERR_CUDA;
  }
  return FKM_OK;
}

constexpr int kSmemBudget = 232448 - 1024;  // opt-in maximum minus alignment slack

}  // namespace

// Shared-memory plan of the assign kernel for D (also used by validation).
bool assign_smem_plan(int D, bool split, int* nA_out, int* nS_out, size_t* smem_out) {
  const int nD = (int)ceil_div(D, KC);
  const long a_bytes = (long)(split ? 2 : 1) * nD * A_CHUNK_BYTES;
  const long s_bytes = B_CHUNK_BYTES;
  const long ctl = (long)((sizeof(SmemCtl) + 127) & ~size_t(127)) + kSaveBytes;
  int nA = 2;
  long nS = (kSmemBudget - ctl - 2 * a_bytes) / s_bytes;
  if (nS < 2) {
    nA = 1;
    nS = (kSmemBudget - ctl - a_bytes) / s_bytes;
  }
  if (nS > 8) nS = 8;
  if (nS < 2) return false;
  if (nA_out) *nA_out = nA;
  if (nS_out) *nS_out = (int)nS;
  if (smem_out) *smem_out = (size_t)(nA * a_bytes + nS * s_bytes + ctl + 1024);
  return true;
}

// Raises the kernels' dynamic shared-memory limit once per device.  Called
// before any stream capture (the attribute call is not a stream operation).
fkm_status assign_prepare() {
  static bool done[64] = {false};
  int dev = 0;
  FKM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && done[dev]) return FKM_OK;
  const int lim = kSmemBudget + 1024;
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<true, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<false, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<true, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<false, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  if (dev >= 0 && dev < 64) done[dev] = true;
  return FKM_OK;
}

fkm_status launch_assign(const AssignArgs& a, cudaStream_t st) {
  int nA = 0, nS = 0;
  size_t smem = 0;
  if (!assign_smem_plan(a.D, a.split, &nA, &nS, &smem)) {
    set_error("D=%d does not fit the assign kernel's shared memory", a.D);
    return FKM_ERR_UNSUPPORTED;
  }
  const int nD = (int)ceil_div(a.D, KC);
  const bool bf16 = a.split || a.dtype == FKM_BF16;
  CUtensorMap tx, txl, tc, tcl;
  // split rows are [hi | lo] with each half padded to a multiple of 8
  // elements, so the lo half starts 16-byte aligned
  const int Dp = (int)round_up(a.D, 8);
  const int Dq = a.split ? 2 * Dp : a.D;
  FKM_TRY(make_map(&tx, a.xq, bf16, a.D, a.N, a.B, a.x_row_elems, KC, BM));
  FKM_TRY(make_map(&tc, a.cq, bf16, a.D, a.Kp, a.B, Dq, KC, BN));
  if (a.split) {
    FKM_TRY(make_map(&txl, static_cast<const uint16_t*>(a.xq) + Dp, true, a.D, a.N, a.B,
                     a.x_row_elems, KC, BM));
    FKM_TRY(make_map(&tcl, static_cast<const uint16_t*>(a.cq) + Dp, true, a.D, a.Kp, a.B, Dq, KC,
                     BN));
  } else {
    txl = tx;
    tcl = tc;
  }
  AssignKParams p;
  p.B = a.B;
  p.N = a.N;
  p.Kp = a.Kp;
  p.nD = nD;
  p.m_tiles = (int)ceil_div(a.N, BM);
  p.k_tiles = a.Kp / BN;
  p.n_work = a.B * p.m_tiles;
  p.nA = nA;
  p.nS = nS;
  p.a_bytes = (uint32_t)((a.split ? 2 : 1) * nD * A_CHUNK_BYTES);
  p.s_bytes = (uint32_t)B_CHUNK_BYTES;
  p.idesc = ptx::umma_idesc_f16(bf16, BM, BN);
  p.cn = a.cn;
  p.xn = a.xn;
  p.ids = a.ids;
  p.status = a.status;
  p.K = a.K;
  p.dist = a.dist;
  const int sms = num_sms();
  const int grid = p.n_work < sms ? p.n_work : sms;
  FKM_TRY(assign_prepare());
  if (a.dist) {
    if (a.split)
      assign_tc_kernel<true, true><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl, p);
    else
      assign_tc_kernel<false, true><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl, p);
  } else if (a.split) {
    assign_tc_kernel<true, false><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl, p);
  } else {
    assign_tc_kernel<false, false><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl, p);
  }
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

}  // namespace fkm
