// FlashAssign on sm_100a: nearest-centroid search without a distance matrix.
//
// "Flash-KMeans: Fast and Memory-Efficient Exact K-Means" summary, section
// "Method" (FlashAssign), and the "Flash-KMeans：快速且内存高效精确K-Means聚类"
// summary, section 方法步骤详情 step (1): tile the points (B_N) and the
// centroids (B_K); per point keep a running (best score, index); per centroid
// tile compute the local B_N x B_K block on chip, take its row extrema and fold
// them into the running state; write the final index once.  The score is
// ||c||^2 - 2 x.c (the same page, section 核心方法: ||x||^2 is constant per
// point and does not change the argmin).
//
// Operands (see prep.cu): centroid offsets q(c - m) from the batch's mean
// centroid m, and a 16-column "bias" slab per centroid holding -n/2 as three
// 16-bit parts, n = ||q(c-m)||^2 + 2 m.q(c-m).  Each point tile is extended by
// a constant slab [a0, a1, a2, 0...] (a = 1, 1, 1 for bf16; 2^15, 2^4, 2^-7
// for fp16, whose parts are scaled to stay in range), so one extra K=16 MMA
// adds the bias and the accumulator holds
//     acc = x.q(c - m) - n/2 = -(score)/2 + (a per-point constant),
// and the nearest centroid is the argmax of acc: the epilogue only compares.
//
// Two kernels share this design.  16-bit points whose point tile fits in
// shared memory (D <= 256) run on CTA pairs (assign_pair_kernel below: one
// MMA of M = 256 spans two SMs).  fp32 points, large D and the comparison
// mode run on single CTAs (assign_tc_kernel), described first.
//
// B200 design (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: the point tile [128 x D] once per work item into
//               one of nA buffers; per centroid tile, 256 x 64 chunks through
//               an nS-stage ring (128-byte swizzle, no multicast), the tile's
//               bias slab (256 x 16, 32-byte swizzle) riding with its first
//               chunk.
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators)
//               and issues tcgen05.mma (M=128, N=256, K=16) from one thread:
//               the bias product, then the point . centroid products.
//   warps 2-9   epilogue, two warpgroups: TMEM lane t = point t of the tile;
//               warpgroup h reads columns [128h, 128h + 128) of every
//               accumulator (four tcgen05.ld in flight, one wait), hands the
//               accumulator back, and keeps the running maximum with 3-input
//               max trees; the chunk that improves it is saved to shared
//               memory so the lowest column holding the maximum is found once
//               per work item.  The two halves are merged per work item.
//               Ties go to the lowest centroid index.
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
#include <cstring>

#include "fkm_internal.cuh"
#include "ptx_sm100.cuh"

namespace fkm {
namespace {

constexpr uint64_t kWaitTimeoutNs = 4000000000ull;  // 4 s
constexpr int AUG_COLS = 16;                             // the bias slab: one K=16 MMA
constexpr int AUG_A_BYTES = BM * AUG_COLS * 2;           // 4 KB, constant per CTA
constexpr int AUG_B_BYTES = BN * AUG_COLS * 2;           // 8 KB per centroid tile
constexpr int STAGE_BYTES = B_CHUNK_BYTES + AUG_B_BYTES; // chunk + bias slot
// Large D (the point tile does not fit shared memory): every stage also
// carries the 128 x 64 point chunk its products need, so the point tile is
// streamed once per centroid tile (from L2 after the first) while the TMEM
// accumulator persists across the D chunks.
constexpr int STAGE_BYTES_STREAM = B_CHUNK_BYTES + A_CHUNK_BYTES + AUG_B_BYTES;
// fp32 points (split hi / lo operands): a stage carries one centroid part (hi
// or lo), the point hi chunk, and for the hi part also the point lo chunk.
constexpr int STAGE_BYTES_STREAM_SPLIT = B_CHUNK_BYTES + 2 * A_CHUNK_BYTES + AUG_B_BYTES;

struct AssignKParams {
  int B, N, Kp, K;
  int nD;          // 64-wide D chunks
  int m_tiles;     // point tiles per batch
  int k_tiles;     // centroid tiles per batch
  int n_work;      // B * m_tiles
  int nA, nS;      // point buffers, centroid stages
  uint32_t a_bytes;
  uint32_t idesc;
  int f16;         // fp16 operands: scaled bias parts
  const float* xn;  // ||x - m||^2, comparison mode only
  int32_t* ids;
  int* status;
  float* dist;     // comparison mode only: the full [B, N, K] distance matrix
};

struct __align__(8) SmemCtl {
  uint64_t a_full[2], a_empty[2];
  uint64_t b_full[8], b_empty[8];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t merge_full, merge_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float2 merge[BM];   // (best, index as float bits) of warpgroup 1
};

// Per epilogue thread, the 32 accumulator values of the chunk that last
// improved its running maximum, with the 16-byte units rotated by lane so the
// predicated stores of a warp hit distinct banks.
constexpr int kSaveBytes = 256 * 32 * 4;

__device__ __forceinline__ float max32(const float (&s)[32]) {
  float m0 = ptx::fmax3(s[0], s[1], s[2]);
  float m1 = ptx::fmax3(s[3], s[4], s[5]);
  float m2 = ptx::fmax3(s[6], s[7], s[8]);
  float m3 = ptx::fmax3(s[9], s[10], s[11]);
  float m4 = ptx::fmax3(s[12], s[13], s[14]);
  float m5 = ptx::fmax3(s[15], s[16], s[17]);
  float m6 = ptx::fmax3(s[18], s[19], s[20]);
  float m7 = ptx::fmax3(s[21], s[22], s[23]);
  float m8 = ptx::fmax3(s[24], s[25], s[26]);
  float m9 = ptx::fmax3(s[27], s[28], s[29]);
  float m10 = fmaxf(s[30], s[31]);
  float n0 = ptx::fmax3(m0, m1, m2);
  float n1 = ptx::fmax3(m3, m4, m5);
  float n2 = ptx::fmax3(m6, m7, m8);
  float n3 = fmaxf(m9, m10);
  return fmaxf(ptx::fmax3(n0, n1, n2), n3);
}

// One 32-column chunk folded into (best, bcol).  A chunk replaces the running
// maximum only when strictly larger; its values are then saved so the lowest
// column holding the maximum is found once per work item (find_first): over
// ascending columns this keeps the lowest centroid index among exact ties.
// Columns at or past K (padding of the last tile) are excluded.
__device__ __forceinline__ void fold_chunk(const uint32_t (&r)[32], int col0, int K, float& best,
                                           int& bcol, float4* save, int rot) {
  float s[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(r[j]);
  if (col0 + 32 > K) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j >= K) s[j] = -INFINITY;
  }
  const float cm = max32(s);
  if (cm > best) {
    best = cm;
    bcol = col0;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      save[k ^ rot] = make_float4(s[4 * k], s[4 * k + 1], s[4 * k + 2], s[4 * k + 3]);
  }
}

// Lowest position j in the saved chunk whose value equals best.
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

// Comparison mode: 32 distances ||x - c_hat||^2 = xv - 2 acc of one row,
// written as 16-byte vectors when the row allows it (K a multiple of 4), so a
// thread's 128 bytes go out whole.
__device__ __forceinline__ void store_dist_chunk(const uint32_t (&r)[32], float* drow, int col0,
                                                 int K, float xv) {
  if (col0 + 32 <= K && (K & 3) == 0) {
    float4* d4 = reinterpret_cast<float4*>(drow + col0);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      d4[k] = make_float4(fmaf(-2.0f, __uint_as_float(r[4 * k]), xv),
                          fmaf(-2.0f, __uint_as_float(r[4 * k + 1]), xv),
                          fmaf(-2.0f, __uint_as_float(r[4 * k + 2]), xv),
                          fmaf(-2.0f, __uint_as_float(r[4 * k + 3]), xv));
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j < K) drow[col0 + j] = fmaf(-2.0f, __uint_as_float(r[j]), xv);
  }
}

// The constant bias slab of a point tile: row r = [a0, a1, a2, 0 ... 0] (16
// values) in the 32-byte swizzle (rows of 32 bytes, 8-row groups of 256
// bytes; the two 16-byte halves of rows 4-7 of a group trade places), the
// layout a K-major tcgen05 operand with SWIZZLE_32B reads.
__device__ __forceinline__ void write_aug_a(uint8_t* base, int f16) {
  if (threadIdx.x >= 2 * BM) return;
  const int r = threadIdx.x >> 1, h = threadIdx.x & 1;
  const int phys = h ^ ((r & 7) >> 2);
  uint4 v = make_uint4(0, 0, 0, 0);
  if (h == 0) {
    uint16_t a0, a1, a2;
    if (f16) {
      a0 = __half_as_ushort(__float2half_rn(32768.0f));
      a1 = __half_as_ushort(__float2half_rn(16.0f));
      a2 = __half_as_ushort(__float2half_rn(0.0078125f));
    } else {
      a0 = a1 = a2 = __bfloat16_as_ushort(__float2bfloat16_rn(1.0f));
    }
    v.x = (uint32_t)a0 | ((uint32_t)a1 << 16);
    v.y = (uint32_t)a2;
  }
  *reinterpret_cast<uint4*>(base + (r >> 3) * 256 + (r & 7) * 32 + phys * 16) = v;
}

// kDist = true is the comparison ("standard") mode: the same tensor-core tiles,
// but the epilogue writes every distance ||x - c_hat||^2 = ||x - m||^2 - 2 acc
// to HBM instead of reducing it, as the pages' baseline assignment does.
template <bool kSplit, bool kDist, bool kStreamA>
__global__ void __launch_bounds__(ASSIGN_THREADS, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap tm_x,    // points (hi part when split)
                     const __grid_constant__ CUtensorMap tm_xl,   // lo part (split only)
                     const __grid_constant__ CUtensorMap tm_c,    // centroid offsets (hi when split)
                     const __grid_constant__ CUtensorMap tm_cl,   // lo part (split only)
                     const __grid_constant__ CUtensorMap tm_aug,  // bias slabs [B][Kp][16]
                     const AssignKParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  constexpr int kStageBytes =
      kStreamA ? (kSplit ? STAGE_BYTES_STREAM_SPLIT : STAGE_BYTES_STREAM) : STAGE_BYTES;
  constexpr int kAugOff =
      kStreamA ? B_CHUNK_BYTES + (kSplit ? 2 : 1) * A_CHUNK_BYTES : B_CHUNK_BYTES;
  uint8_t* a_base = smem;
  uint8_t* aug_a = a_base + (kStreamA ? 0 : (size_t)p.nA * p.a_bytes);
  uint8_t* b_base = aug_a + AUG_A_BYTES;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(b_base + (size_t)p.nS * kStageBytes);
  float4* save_base = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(ctl) +
                                                ((sizeof(SmemCtl) + 127) & ~size_t(127)));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &ctl->abort;

  write_aug_a(aug_a, p.f16);
  // the generic-proxy stores above are read by the tensor cores (async proxy)
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
  const int nQ = p.nD * (kSplit ? 2 : 1);   // stages per centroid tile
  // the set-up above touched only this CTA's shared memory and TMEM; global
  // memory waits for the previous kernel of the stream
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_x);
      ptx::prefetch_tmap(&tm_c);
      ptx::prefetch_tmap(&tm_aug);
      if (kSplit) {
        ptx::prefetch_tmap(&tm_xl);
        ptx::prefetch_tmap(&tm_cl);
      }
      uint32_t a_arms = 0, s_arms = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.n_work && ok; w += gridDim.x) {
        const int b = w / p.m_tiles, mt = w % p.m_tiles;
        if (!kStreamA) {
          const int ab = a_arms % p.nA;
          const uint32_t apar = ((a_arms / p.nA) & 1) ^ 1;
          if (!ptx::mbar_wait_bounded(&ctl->a_empty[ab], apar, abort_flag, p.status, ST_TIMEOUT,
                                      kWaitTimeoutNs)) { ok = false; break; }
          ptx::mbar_arrive_expect_tx(&ctl->a_full[ab], p.a_bytes);
          uint8_t* abuf = a_base + (size_t)ab * p.a_bytes;
          for (int dc = 0; dc < p.nD; ++dc) {
            ptx::tma_load_3d(abuf + dc * A_CHUNK_BYTES, &tm_x, &ctl->a_full[ab], dc * KC, mt * BM,
                             b);
            if (kSplit)
              ptx::tma_load_3d(abuf + (p.nD + dc) * A_CHUNK_BYTES, &tm_xl, &ctl->a_full[ab],
                               dc * KC, mt * BM, b);
          }
          ++a_arms;
        }
        for (int kt = 0; kt < p.k_tiles && ok; ++kt) {
          // one stage per 64-wide chunk (split operands: hi and lo in
          // consecutive stages); the tile's bias slab rides with its first chunk
          for (int q = 0; q < nQ; ++q) {
            const int dc = kSplit ? (q >> 1) : q;
            const int sb = s_arms % p.nS;
            const uint32_t spar = ((s_arms / p.nS) & 1) ^ 1;
            if (!ptx::mbar_wait_bounded(&ctl->b_empty[sb], spar, abort_flag, p.status, ST_TIMEOUT,
                                        kWaitTimeoutNs)) { ok = false; break; }
            // streamed points: the hi part of a split chunk also needs the lo points
            const bool lo_pts = kStreamA && kSplit && !(q & 1);
            ptx::mbar_arrive_expect_tx(&ctl->b_full[sb],
                                       B_CHUNK_BYTES + (kStreamA ? A_CHUNK_BYTES : 0) +
                                           (lo_pts ? A_CHUNK_BYTES : 0) +
                                           (q == 0 ? AUG_B_BYTES : 0));
            uint8_t* sbuf = b_base + (size_t)sb * kStageBytes;
            ptx::tma_load_3d(sbuf, (kSplit && (q & 1)) ? &tm_cl : &tm_c, &ctl->b_full[sb],
                             dc * KC, kt * BN, b);
            if (kStreamA)   // the point chunk these products need
              ptx::tma_load_3d(sbuf + B_CHUNK_BYTES, &tm_x, &ctl->b_full[sb], dc * KC, mt * BM, b);
            if (lo_pts)
              ptx::tma_load_3d(sbuf + B_CHUNK_BYTES + A_CHUNK_BYTES, &tm_xl, &ctl->b_full[sb],
                               dc * KC, mt * BM, b);
            if (q == 0)
              ptx::tma_load_3d(sbuf + kAugOff, &tm_aug, &ctl->b_full[sb], 0, kt * BN, b);
            ++s_arms;
          }
        }
      }
      // Drain: every buffer's most recent load must have landed before exit.
      for (uint32_t i = 0; !kStreamA && i < (uint32_t)p.nA && i < a_arms; ++i) {
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
      const uint32_t aug_a_addr = ptx::smem_u32(aug_a);
      uint32_t a_uses = 0, s_uses = 0, acc_uses = 0;
      bool ok = true;
      bool issued = false;
      for (int w = blockIdx.x; w < p.n_work && ok; w += gridDim.x) {
        const int ab = kStreamA ? 0 : a_uses % p.nA;
        if (!kStreamA) {
          if (!ptx::mbar_wait_bounded(&ctl->a_full[ab], (a_uses / p.nA) & 1, abort_flag,
                                      p.status, ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
          ptx::tc_fence_after();
        }
        const uint32_t a_addr = ptx::smem_u32(a_base + (size_t)ab * p.a_bytes);
        for (int kt = 0; kt < p.k_tiles && ok; ++kt) {
          const int acc = acc_uses & 1;
          if (!ptx::mbar_wait_bounded(&ctl->acc_empty[acc], ((acc_uses >> 1) & 1) ^ 1, abort_flag,
                                      p.status, ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          for (int q = 0; q < nQ; ++q) {
            const int dc = kSplit ? (q >> 1) : q;
            const int sb = s_uses % p.nS;
            if (!ptx::mbar_wait_bounded(&ctl->b_full[sb], (s_uses / p.nS) & 1, abort_flag,
                                        p.status, ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t b_addr = ptx::smem_u32(b_base + (size_t)sb * kStageBytes);
            const uint32_t xa = kStreamA ? b_addr + B_CHUNK_BYTES : a_addr + dc * A_CHUNK_BYTES;
            if (q == 0)   // the bias product starts the tile's accumulation
              ptx::mma_f16_ss(d_tmem, ptx::umma_desc_sw32(aug_a_addr),
                              ptx::umma_desc_sw32(b_addr + kAugOff), p.idesc, 0u);
            if (!(kSplit && (q & 1))) {
              // xh . ch (or x . q(c - m))
#pragma unroll
              for (int k = 0; k < KC / 16; ++k)
                ptx::mma_f16_ss(d_tmem, ptx::umma_desc_sw128(xa + 32 * k),
                                ptx::umma_desc_sw128(b_addr + 32 * k), p.idesc, 1u);
              if (kSplit) {   // xl . ch
                const uint32_t xl = kStreamA ? b_addr + B_CHUNK_BYTES + A_CHUNK_BYTES
                                             : a_addr + (p.nD + dc) * A_CHUNK_BYTES;
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
        if (!kStreamA) {
          ptx::mma_commit(&ctl->a_empty[ab]);
          ++a_uses;
        }
      }
      // Drain: all MMAs this thread issued must finish before TMEM is freed.
      if (issued) {
        ptx::mma_commit(&ctl->drain);
        ptx::mbar_wait_bounded(&ctl->drain, 0, abort_flag, p.status, ST_TIMEOUT, kWaitTimeoutNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                  // epilogue warp 0..7
    const int half = ew >> 2;                 // columns [128*half, 128*half + 128) of a tile
    const int quad = warp & 3;                // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;         // point within the tile
    const int rot = lane & 7;
    float4* save = save_base + (size_t)(ew * 32 + lane) * 8;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    uint32_t acc_uses = 0, items = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < p.n_work && ok; w += gridDim.x, ++items) {
      const int b = w / p.m_tiles, mt = w % p.m_tiles;
      const int gi = mt * BM + row;
      float best = -INFINITY;
      int bcol = 0;
      for (int kt = 0; kt < p.k_tiles; ++kt) {
        const int acc = acc_uses & 1;
        const uint32_t par = (acc_uses >> 1) & 1;
        if (!ptx::mbar_wait_bounded(&ctl->acc_full[acc], par, abort_flag, p.status, ST_TIMEOUT,
                                    kWaitTimeoutNs)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t taddr = lane_addr + (uint32_t)(acc * BN + half * 128);
        const int colb = kt * BN + half * 128;
        // all 128 of this warp's columns in flight at once, one wait, then the
        // accumulator goes straight back to the MMA warp
        uint32_t r0[32], r1[32], r2[32], r3[32];
        ptx::tmem_ld32(taddr, r0);
        ptx::tmem_ld32(taddr + 32, r1);
        ptx::tmem_ld32(taddr + 64, r2);
        ptx::tmem_ld32(taddr + 96, r3);
        ptx::tmem_wait_ld128(r0, r1, r2, r3);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&ctl->acc_empty[acc]);
        ++acc_uses;
        if (kDist) {
          if (gi < p.N) {
            const float xv = p.xn[(size_t)b * p.N + gi];
            float* drow = p.dist + ((size_t)b * p.N + gi) * p.K;
            store_dist_chunk(r0, drow, colb, p.K, xv);
            store_dist_chunk(r1, drow, colb + 32, p.K, xv);
            store_dist_chunk(r2, drow, colb + 64, p.K, xv);
            store_dist_chunk(r3, drow, colb + 96, p.K, xv);
          }
          continue;
        }
        fold_chunk(r0, colb, p.K, best, bcol, save, rot);
        fold_chunk(r1, colb + 32, p.K, best, bcol, save, rot);
        fold_chunk(r2, colb + 64, p.K, best, bcol, save, rot);
        fold_chunk(r3, colb + 96, p.K, best, bcol, save, rot);
      }
      if (!ok) break;
      if (kDist) continue;
      const int idx = best > -INFINITY ? bcol + find_first(save, rot, best) : 0;
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
        const int fidx = (o.x > best || (o.x == best && oidx < idx)) ? oidx : idx;
        if (gi < p.N && fkm_in_range(fidx, p.K, p.status)) p.ids[(size_t)b * p.N + gi] = fidx;
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

// ------------------------------------------------------------------ CTA pairs
// The main path (16-bit points, point tile resident in shared memory): a
// cluster of two CTAs on neighbouring SMs shares every MMA (tcgen05
// cta_group::2, M = 256).  CTA r of the pair holds rows [256 w + 128 r, +128)
// of work item w and rows [128 r, +128) of every 256-centroid tile; the even
// CTA issues the MMAs, and each CTA's TMEM receives its own 128 x 256
// accumulator, which its own epilogue warps reduce as above.  Per SM this
// halves the centroid bytes streamed from L2 and the B-operand bytes the
// tensor cores read from shared memory per MMA: with one CTA per tile those
// reads plus the TMA refills exceed the SM's shared-memory bandwidth and
// hold the tensor pipe well below its peak.
//
// Synchronisation across the pair: TMA loads of both CTAs complete on the
// even CTA's "full" barriers (cta_group::2 form, no multicast), whose
// expected byte count covers both halves; tcgen05.commit with a two-CTA mask
// arrives on the "empty" and accumulator-full barriers of both CTAs; each
// epilogue warp of either CTA arrives on the even CTA's accumulator-empty
// barrier (16 arrivals) once its TMEM reads are done.  Every wait is bounded
// as in the single-CTA kernel; a cluster barrier precedes the TMEM release.
constexpr int PAIR_BH = BN / 2;                          // centroid rows per CTA
constexpr int PAIR_B_CHUNK = PAIR_BH * KC * 2;           // 16 KB
constexpr int PAIR_AUG_B = PAIR_BH * AUG_COLS * 2;       // 4 KB
constexpr int PAIR_STAGE = PAIR_B_CHUNK + PAIR_AUG_B;    // 20 KB (1024-byte multiple)
constexpr int PAIR_ROWS = 2 * BM;                        // points per work item

struct __align__(8) PairCtl {
  uint64_t a_full[2], a_empty[2];
  uint64_t b_full[8], b_empty[8];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t merge_full, merge_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float2 merge[BM];   // (best, index as float bits) of warpgroup 1
};

// Two adjacent chunks (64 columns from col0) folded at once: the chunk
// holding the larger maximum (the lower one on a tie, so the lowest column
// still wins) replaces the saved chunk when it beats the running maximum.
// One decision per 64 columns halves the copies a warp makes, which every
// lane pays for when any lane improves.
__device__ __forceinline__ void fold_pair_reg(const uint32_t (&r0)[32], const uint32_t (&r1)[32],
                                              int col0, int K, float& best, int& bcol,
                                              float (&sv)[32]) {
  float s0[32], s1[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    s0[j] = __uint_as_float(r0[j]);
    s1[j] = __uint_as_float(r1[j]);
  }
  if (col0 + 64 > K) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (col0 + j >= K) s0[j] = -INFINITY;
      if (col0 + 32 + j >= K) s1[j] = -INFINITY;
    }
  }
  const float cm0 = max32(s0), cm1 = max32(s1);
  const float bm = fmaxf(cm0, cm1);
  if (bm > best) {
    best = bm;
    const bool first = cm0 >= cm1;
    bcol = first ? col0 : col0 + 32;
#pragma unroll
    for (int j = 0; j < 32; ++j) sv[j] = first ? s0[j] : s1[j];
  }
}

__device__ __forceinline__ int find_first_reg(const float (&sv)[32], float best) {
  uint32_t mask = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) mask |= (uint32_t)(sv[j] == best) << j;
  return mask ? __ffs(mask) - 1 : 0;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(ASSIGN_THREADS, 1)
    assign_pair_kernel(const __grid_constant__ CUtensorMap tm_x,    // points, box 64 x 128
                       const __grid_constant__ CUtensorMap tm_c,    // centroid offsets, box 64 x 128
                       const __grid_constant__ CUtensorMap tm_aug,  // bias slabs, box 16 x 128
                       const AssignKParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* a_base = smem;
  uint8_t* aug_a = a_base + (size_t)p.nA * p.a_bytes;
  uint8_t* b_base = aug_a + AUG_A_BYTES;
  PairCtl* ctl = reinterpret_cast<PairCtl*>(b_base + (size_t)p.nS * PAIR_STAGE);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t cid = ptx::cluster_id_x(), ncl = ptx::n_clusters_x();
  volatile int* abort_flag = &ctl->abort;

  write_aug_a(aug_a, p.f16);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
      ptx::mbar_init(&ctl->acc_empty[i], 16);   // 8 epilogue warps in each CTA
    }
    ptx::mbar_init(&ctl->merge_full, 128);
    ptx::mbar_init(&ctl->merge_empty, 128);
    ptx::mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(&ctl->tmem_base, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncwarp();
  // both CTAs' barriers exist and their TMEM is allocated before any
  // cross-CTA arrival or MMA
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  // the set-up above touched only the pair's shared memory and TMEM; global
  // memory waits for the previous kernel of the stream
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producers (both CTAs)
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_x);
      ptx::prefetch_tmap(&tm_c);
      ptx::prefetch_tmap(&tm_aug);
      uint32_t a_arms = 0, s_arms = 0;
      uint32_t ab = 0, a_ph = 0, sb = 0, s_ph = 0;   // ring positions, as in the issuer
      bool ok = true;
      for (int w = (int)cid; w < p.n_work && ok; w += (int)ncl) {
        const int b = w / p.m_tiles, mt = w % p.m_tiles;
        const int row0 = mt * PAIR_ROWS + (int)rank * BM;
        if (!ptx::mbar_wait_bounded_cl(&ctl->a_empty[ab], a_ph ^ 1, abort_flag, p.status,
                                       ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
        if (leader) ptx::mbar_arrive_expect_tx(&ctl->a_full[ab], 2 * p.a_bytes);
        const uint32_t afull = ptx::mapa_rank(&ctl->a_full[ab], 0);
        uint8_t* abuf = a_base + (size_t)ab * p.a_bytes;
        for (int dc = 0; dc < p.nD; ++dc)
          ptx::tma_load_3d_pair(abuf + dc * A_CHUNK_BYTES, &tm_x, afull, dc * KC, row0, b);
        ++a_arms;
        if (++ab == (uint32_t)p.nA) { ab = 0; a_ph ^= 1; }
        for (int kt = 0; kt < p.k_tiles && ok; ++kt) {
          const int crow = kt * BN + (int)rank * PAIR_BH;
          for (int q = 0; q < p.nD; ++q) {
            if (!ptx::mbar_wait_bounded_cl(&ctl->b_empty[sb], s_ph ^ 1, abort_flag, p.status,
                                           ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
            if (leader)
              ptx::mbar_arrive_expect_tx(&ctl->b_full[sb],
                                         2 * (PAIR_B_CHUNK + (q == 0 ? PAIR_AUG_B : 0)));
            const uint32_t bfull = ptx::mapa_rank(&ctl->b_full[sb], 0);
            uint8_t* sbuf = b_base + (size_t)sb * PAIR_STAGE;
            ptx::tma_load_3d_pair(sbuf, &tm_c, bfull, q * KC, crow, b);
            if (q == 0) ptx::tma_load_3d_pair(sbuf + PAIR_B_CHUNK, &tm_aug, bfull, 0, crow, b);
            ++s_arms;
            if (++sb == (uint32_t)p.nS) { sb = 0; s_ph ^= 1; }
          }
        }
      }
      // Drain: the last use of every buffer was consumed by the MMAs (which
      // also means its loads landed) before this CTA may leave.
      for (uint32_t i = 0; i < (uint32_t)p.nA && i < a_arms; ++i) {
        const uint32_t last = i + p.nA * ((a_arms - 1 - i) / p.nA);
        ptx::mbar_wait_bounded_cl(&ctl->a_empty[i], (last / p.nA) & 1, abort_flag, p.status,
                                  ST_TIMEOUT, kWaitTimeoutNs);
      }
      for (uint32_t i = 0; i < (uint32_t)p.nS && i < s_arms; ++i) {
        const uint32_t last = i + p.nS * ((s_arms - 1 - i) / p.nS);
        ptx::mbar_wait_bounded_cl(&ctl->b_empty[i], (last / p.nS) & 1, abort_flag, p.status,
                                  ST_TIMEOUT, kWaitTimeoutNs);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    // One thread feeds the tensor pipe, and an M = 256, N = 256, K = 16 MMA
    // occupies it for only ~128 cycles, so this loop keeps its own work per
    // MMA to a few instructions: ring indices and phases advance without
    // divisions, and every operand descriptor is a base descriptor plus the
    // operand's byte offset >> 4 (the start-address field, bits 0-13, cannot
    // carry below 256 KB).  A division or a rebuilt descriptor per MMA was
    // enough to leave the pipe idle half of the time.
    if (leader && lane == 0) {
      const uint64_t d_aug_a = ptx::umma_desc_sw32(ptx::smem_u32(aug_a));
      const uint64_t d_a0 = ptx::umma_desc_sw128(ptx::smem_u32(a_base));
      const uint64_t d_b0 = ptx::umma_desc_sw128(ptx::smem_u32(b_base));
      const uint64_t d_aug_b0 = ptx::umma_desc_sw32(ptx::smem_u32(b_base + PAIR_B_CHUNK));
      constexpr uint32_t kStageStep = PAIR_STAGE >> 4, kChunkStep = A_CHUNK_BYTES >> 4;
      const uint32_t a_step = p.a_bytes >> 4;
      uint32_t ab = 0, a_ph = 0, sb = 0, s_ph = 0, acc = 0, acc_ph = 0;
      bool ok = true, issued = false;
      for (int w = (int)cid; w < p.n_work && ok; w += (int)ncl) {
        if (!ptx::mbar_wait_bounded_cl(&ctl->a_full[ab], a_ph, abort_flag, p.status, ST_TIMEOUT,
                                       kWaitTimeoutNs)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint64_t d_a = d_a0 + ab * a_step;
        for (int kt = 0; kt < p.k_tiles && ok; ++kt) {
          if (!ptx::mbar_wait_bounded_cl(&ctl->acc_empty[acc], acc_ph ^ 1, abort_flag, p.status,
                                         ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * BN;
          for (int q = 0; q < p.nD; ++q) {
            if (!ptx::mbar_wait_bounded_cl(&ctl->b_full[sb], s_ph, abort_flag, p.status,
                                           ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint64_t d_b = d_b0 + sb * kStageStep;
            if (q == 0)   // the bias product starts the tile's accumulation
              ptx::mma_f16_ss_pair(d_tmem, d_aug_a, d_aug_b0 + sb * kStageStep, p.idesc, 0u);
            const uint64_t d_aq = d_a + q * kChunkStep;
#pragma unroll
            for (int k = 0; k < KC / 16; ++k)   // K = 16 steps are 32 bytes apart
              ptx::mma_f16_ss_pair(d_tmem, d_aq + 2 * k, d_b + 2 * k, p.idesc, 1u);
            issued = true;
            ptx::mma_commit_pair_mc(&ctl->b_empty[sb], 0x3);
            if (++sb == (uint32_t)p.nS) { sb = 0; s_ph ^= 1; }
          }
          if (!ok) break;
          ptx::mma_commit_pair_mc(&ctl->acc_full[acc], 0x3);
          if (++acc == 2) { acc = 0; acc_ph ^= 1; }
        }
        if (!ok) break;
        ptx::mma_commit_pair_mc(&ctl->a_empty[ab], 0x3);
        if (++ab == (uint32_t)p.nA) { ab = 0; a_ph ^= 1; }
      }
      // Drain: all MMAs issued must finish before TMEM is freed.
      if (issued) {
        ptx::mma_commit_pair_mc(&ctl->drain, 0x1);
        ptx::mbar_wait_bounded_cl(&ctl->drain, 0, abort_flag, p.status, ST_TIMEOUT,
                                  kWaitTimeoutNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int ew = warp - 2;
    const int half = ew >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quad * 32) << 16);
    const uint32_t acc_empty_cl[2] = {ptx::mapa_rank(&ctl->acc_empty[0], 0),
                                      ptx::mapa_rank(&ctl->acc_empty[1], 0)};
    uint32_t acc_uses = 0, items = 0;
    bool ok = true;
    float sv[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) sv[j] = -INFINITY;
    for (int w = (int)cid; w < p.n_work && ok; w += (int)ncl, ++items) {
      const int b = w / p.m_tiles, mt = w % p.m_tiles;
      const int gi = mt * PAIR_ROWS + (int)rank * BM + row;
      float best = -INFINITY;
      int bcol = 0;
      for (int kt = 0; kt < p.k_tiles; ++kt) {
        const int acc = acc_uses & 1;
        const uint32_t par = (acc_uses >> 1) & 1;
        if (!ptx::mbar_wait_bounded_cl(&ctl->acc_full[acc], par, abort_flag, p.status,
                                       ST_TIMEOUT, kWaitTimeoutNs)) { ok = false; break; }
        ptx::tc_fence_after();
        const uint32_t taddr = lane_addr + (uint32_t)(acc * BN + half * 128);
        const int colb = kt * BN + half * 128;
        // two batches of 64 columns keep the live registers within the
        // 320-thread block's budget (the improving chunk is kept in
        // registers); the accumulator goes back once the second batch landed
        uint32_t r0[32], r1[32];
        ptx::tmem_ld32(taddr, r0);
        ptx::tmem_ld32(taddr + 32, r1);
        ptx::tmem_wait_ld64(r0, r1);
        fold_pair_reg(r0, r1, colb, p.K, best, bcol, sv);
        __syncwarp();   // the folds branch per lane; tcgen05.ld is warp-wide
        ptx::tmem_ld32(taddr + 64, r0);
        ptx::tmem_ld32(taddr + 96, r1);
        ptx::tmem_wait_ld64(r0, r1);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(acc_empty_cl[acc]);
        ++acc_uses;
        fold_pair_reg(r0, r1, colb + 64, p.K, best, bcol, sv);
      }
      if (!ok) break;
      const int idx = best > -INFINITY ? bcol + find_first_reg(sv, best) : 0;
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
        const int fidx = (o.x > best || (o.x == best && oidx < idx)) ? oidx : idx;
        if (gi < p.N && fkm_in_range(fidx, p.K, p.status)) p.ids[(size_t)b * p.N + gi] = fidx;
      }
    }
  }

  ptx::tc_fence_before();
  __syncwarp();
  // both CTAs are done with TMEM and with each other's barriers
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
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
// row_elems; the box is box_cols x box_rows x 1.  Elements outside
// [cols) x [rows) read as zero.
fkm_status make_map(CUtensorMap* m, const void* base, bool bf16, int cols, int rows, int batches,
                    int row_elems, int box_cols, int box_rows,
                    CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
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
                   swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
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
// The point tile stays resident (double-buffered when it fits) up to D = 256
// (fp32 points: 128); beyond that it is streamed chunk by chunk with the
// centroids.
bool assign_smem_plan(int D, bool split, int* nA_out, int* nS_out, size_t* smem_out,
                      bool* stream_out) {
  const int nD = (int)ceil_div(D, KC);
  const long a_bytes = (long)(split ? 2 : 1) * nD * A_CHUNK_BYTES;
  const long ctl = (long)((sizeof(SmemCtl) + 127) & ~size_t(127)) + kSaveBytes + AUG_A_BYTES;
  int nA = 0;
  long nS = 0, s_bytes = STAGE_BYTES;
  bool stream = false;
  if (D <= (split ? 128 : 256)) {
    nA = 2;
    nS = (kSmemBudget - ctl - 2 * a_bytes) / s_bytes;
    if (nS < 2) {
      nA = 1;
      nS = (kSmemBudget - ctl - a_bytes) / s_bytes;
    }
  } else if (D <= ASSIGN_MAX_D) {
    stream = true;
    s_bytes = split ? STAGE_BYTES_STREAM_SPLIT : STAGE_BYTES_STREAM;
    nS = (kSmemBudget - ctl) / s_bytes;
  }
  if (nS > 8) nS = 8;
  if (nS < 2) return false;
  if (nA_out) *nA_out = nA;
  if (nS_out) *nS_out = (int)nS;
  if (smem_out) *smem_out = (size_t)(nA * a_bytes + nS * s_bytes + ctl + 1024);
  if (stream_out) *stream_out = stream;
  return true;
}

// Shared-memory plan of the CTA-pair kernel (16-bit points, D <= 256).
static bool assign_pair_plan(int D, int* nA_out, int* nS_out, size_t* smem_out) {
  if (D > 256) return false;
  const int nD = (int)ceil_div(D, KC);
  const long a_bytes = (long)nD * A_CHUNK_BYTES;
  const long ctl = (long)((sizeof(PairCtl) + 127) & ~size_t(127)) + AUG_A_BYTES;
  int nA = 2;
  long nS = (kSmemBudget - ctl - 2 * a_bytes) / PAIR_STAGE;
  if (nS < 3) {
    nA = 1;
    nS = (kSmemBudget - ctl - a_bytes) / PAIR_STAGE;
  }
  if (nS > 8) nS = 8;
  if (nS < 2) return false;
  if (nA_out) *nA_out = nA;
  if (nS_out) *nS_out = (int)nS;
  if (smem_out) *smem_out = (size_t)(nA * a_bytes + nS * PAIR_STAGE + ctl + 1024);
  return true;
}

// Clusters of two the pair kernel keeps resident at once (per device).
static int pair_clusters[64] = {0};

// Raises the kernels' dynamic shared-memory limit once per device.  Called
// before any stream capture (the attribute call is not a stream operation).
fkm_status assign_prepare() {
  static bool done[64] = {false};
  int dev = 0;
  FKM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && done[dev]) return FKM_OK;
  const int lim = kSmemBudget + 1024;
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<true, false, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<false, false, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<true, true, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<false, true, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<false, false, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<false, true, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<true, false, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_tc_kernel<true, true, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  FKM_CUDA_TRY(cudaFuncSetAttribute(assign_pair_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, lim));
  // resident clusters of the pair kernel at its largest shared-memory plan
  {
    size_t smem = 0;
    assign_pair_plan(64, nullptr, nullptr, &smem);
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(2 * (num_sms() / 2)), 1, 1);
    cfg.blockDim = dim3(ASSIGN_THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)lim;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, assign_pair_kernel, &cfg) != cudaSuccess ||
        n <= 0) {
      cudaGetLastError();
      n = num_sms() / 2;
    }
    if (dev >= 0 && dev < 64) pair_clusters[dev] = n;
  }
  if (dev >= 0 && dev < 64) done[dev] = true;
  return FKM_OK;
}

static fkm_status launch_assign_pair(const AssignArgs& a, cudaStream_t st) {
  int nA = 0, nS = 0;
  size_t smem = 0;
  assign_pair_plan(a.D, &nA, &nS, &smem);
  const int nD = (int)ceil_div(a.D, KC);
  const bool bf16 = a.dtype == FKM_BF16;
  CUtensorMap tx, tc, taug;
  FKM_TRY(make_map(&tx, a.xq, bf16, a.D, a.N, a.B, a.x_row_elems, KC, BM));
  FKM_TRY(make_map(&tc, a.cq, bf16, a.D, a.Kp, a.B, a.D, KC, PAIR_BH));
  FKM_TRY(make_map(&taug, a.caug, bf16, AUG_COLS, a.Kp, a.B, AUG_COLS, AUG_COLS, PAIR_BH,
                   CU_TENSOR_MAP_SWIZZLE_32B));
  AssignKParams p;
  memset(&p, 0, sizeof(p));
  p.B = a.B;
  p.N = a.N;
  p.Kp = a.Kp;
  p.K = a.K;
  p.nD = nD;
  p.m_tiles = (int)ceil_div(a.N, PAIR_ROWS);
  p.k_tiles = a.Kp / BN;
  p.n_work = a.B * p.m_tiles;
  p.nA = nA;
  p.nS = nS;
  p.a_bytes = (uint32_t)(nD * A_CHUNK_BYTES);
  p.idesc = ptx::umma_idesc_f16(bf16, 2 * BM, BN);
  p.f16 = bf16 ? 0 : 1;
  p.ids = a.ids;
  p.status = a.status;
  FKM_TRY(assign_prepare());
  int dev = 0;
  FKM_CUDA_TRY(cudaGetDevice(&dev));
  int clusters = (dev >= 0 && dev < 64 && pair_clusters[dev] > 0) ? pair_clusters[dev]
                                                                    : num_sms() / 2;
  if (clusters > p.n_work) clusters = p.n_work;
  FKM_CUDA_TRY(launch_pdl(assign_pair_kernel, dim3(2 * clusters), dim3(ASSIGN_THREADS), smem, st,
                          tx, tc, taug, p));
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

fkm_status launch_assign(const AssignArgs& a, cudaStream_t st) {
  // 16-bit points with the point tile resident in shared memory: CTA pairs
  if (!a.split && !a.dist && assign_pair_plan(a.D, nullptr, nullptr, nullptr))
    return launch_assign_pair(a, st);
  int nA = 0, nS = 0;
  size_t smem = 0;
  bool stream = false;
  if (!assign_smem_plan(a.D, a.split, &nA, &nS, &smem, &stream)) {
    set_error("D=%d does not fit the assign kernel's shared memory", a.D);
    return FKM_ERR_UNSUPPORTED;
  }
  const int nD = (int)ceil_div(a.D, KC);
  const bool bf16 = a.split || a.dtype == FKM_BF16;
  CUtensorMap tx, txl, tc, tcl, taug;
  // split rows are [hi | lo] with each half padded to a multiple of 8
  // elements, so the lo half starts 16-byte aligned
  const int Dp = (int)round_up(a.D, 8);
  const int Dq = a.split ? 2 * Dp : a.D;
  FKM_TRY(make_map(&tx, a.xq, bf16, a.D, a.N, a.B, a.x_row_elems, KC, BM));
  FKM_TRY(make_map(&tc, a.cq, bf16, a.D, a.Kp, a.B, Dq, KC, BN));
  FKM_TRY(make_map(&taug, a.caug, bf16, AUG_COLS, a.Kp, a.B, AUG_COLS, AUG_COLS, BN,
                   CU_TENSOR_MAP_SWIZZLE_32B));
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
  p.K = a.K;
  p.nD = nD;
  p.m_tiles = (int)ceil_div(a.N, BM);
  p.k_tiles = a.Kp / BN;
  p.n_work = a.B * p.m_tiles;
  p.nA = nA;
  p.nS = nS;
  p.a_bytes = (uint32_t)((a.split ? 2 : 1) * nD * A_CHUNK_BYTES);
  p.idesc = ptx::umma_idesc_f16(bf16, BM, BN);
  p.f16 = bf16 ? 0 : 1;
  p.xn = a.xn;
  p.ids = a.ids;
  p.status = a.status;
  p.dist = a.dist;
  const int sms = num_sms();
  const int grid = p.n_work < sms ? p.n_work : sms;
  FKM_TRY(assign_prepare());
  if (stream) {
    if (a.split && a.dist)
      assign_tc_kernel<true, true, true><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl,
                                                                             taug, p);
    else if (a.split)
      assign_tc_kernel<true, false, true><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl,
                                                                              taug, p);
    else if (a.dist)
      assign_tc_kernel<false, true, true><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl,
                                                                              taug, p);
    else
      assign_tc_kernel<false, false, true><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl,
                                                                               taug, p);
  } else if (a.dist) {
    if (a.split)
      assign_tc_kernel<true, true, false><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl,
                                                                              taug, p);
    else
      assign_tc_kernel<false, true, false><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl,
                                                                               taug, p);
  } else if (a.split) {
    assign_tc_kernel<true, false, false><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl,
                                                                             taug, p);
  } else {
    assign_tc_kernel<false, false, false><<<grid, ASSIGN_THREADS, smem, st>>>(tx, txl, tc, tcl,
                                                                              taug, p);
  }
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

}  // namespace fkm
