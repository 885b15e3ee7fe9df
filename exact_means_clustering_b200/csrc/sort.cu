// Stable device argsort of the 1-D assignment vector.
//
// Sort-Inverse Update starts by argsorting the assignment vector so equal
// cluster ids form contiguous runs, giving the inverse mapping sorted_idx
// ("Flash-KMeans：快速且内存高效精确K-Means聚类" summary, sections 前置知识 /
// argsort与分段规约 and 方法步骤详情 step (2)).  Keys are key = b*K + id (so
// batches stay apart); values are the row indices b*N + i.
//
// LSD radix sort, 8-bit digits, as many passes as the key width needs
// (1 for B*K < 256, 2 up to 65536).  Per pass:
//   upsweep    tile histograms (4096 keys per 256-thread tile), digit-major
//   scan       exclusive scan of the histogram matrix: global base per
//              (digit, tile)
//   downsweep  stable rank of every key inside its tile (warp match_any
//              ranking), keys and values staged in shared memory in sorted
//              order, then written out in contiguous runs per digit.
// The first pass forms the keys from the ids on the fly and validates them:
// an id outside [0, K) sets ST_BAD_ID and gets the sentinel key B*K, which
// sorts after every real key.
#include "fkm_internal.cuh"

namespace fkm {
namespace {

constexpr int kScanBlock = 1024;
constexpr int kScanItems = 4;
constexpr int kScanChunk = kScanBlock * kScanItems;

struct KeySrc {
  const int32_t* keys;  // pass >= 1: previous pass output
  const int32_t* vals;
  const int32_t* ids;   // pass 0: ids
  int N, K;             // pass 0 key formation
  int sentinel;         // B*K
  int* status;
};

template <bool kFirst>
__device__ __forceinline__ void load_key(const KeySrc& s, int64_t j, int32_t& key, int32_t& val) {
  if (kFirst) {
    const int32_t id = s.ids[j];
    const int32_t b = (int32_t)(j / s.N);
    if (id < 0 || id >= s.K) {
      atomicOr(s.status, ST_BAD_ID);
      key = s.sentinel;
    } else {
      key = b * s.K + id;
    }
    val = (int32_t)j;
  } else {
    key = s.keys[j];
    val = s.vals[j];
  }
}

template <bool kFirst>
__global__ void __launch_bounds__(SORT_THREADS) radix_upsweep(KeySrc s, int64_t n, int shift,
                                                              int n_tiles, uint32_t* hist) {
  __shared__ uint32_t h[SORT_THREADS / 32][RADIX_BINS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < (SORT_THREADS / 32) * RADIX_BINS; i += SORT_THREADS)
    (&h[0][0])[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * SORT_TILE;
#pragma unroll 4
  for (int it = 0; it < SORT_ITEMS; ++it) {
    const int64_t j = base + (int64_t)it * SORT_THREADS + threadIdx.x;
    int digit = RADIX_BINS;  // out of range: matches nothing real
    if (j < n) {
      int32_t key, val;
      load_key<kFirst>(s, j, key, val);
      digit = (key >> shift) & (RADIX_BINS - 1);
    }
    const unsigned peers = __match_any_sync(0xffffffffu, digit);
    if (digit < RADIX_BINS && lane == __ffs(peers) - 1) atomicAdd(&h[warp][digit], __popc(peers));
  }
  __syncthreads();
  for (int d = threadIdx.x; d < RADIX_BINS; d += SORT_THREADS) {
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < SORT_THREADS / 32; ++w) t += h[w][d];
    hist[(size_t)d * n_tiles + blockIdx.x] = t;
  }
}

// --- device-wide exclusive scan of uint32 (three phases) ---
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* sh_warp,
                                                         uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < nw ? sh_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) sh_warp[lane] = w;
  }
  __syncthreads();
  const uint32_t wpre = warp > 0 ? sh_warp[warp - 1] : 0;
  if (total) *total = sh_warp[nw - 1];
  __syncthreads();
  return wpre + x - v;
}

__global__ void __launch_bounds__(kScanBlock) scan_reduce(const uint32_t* in, int64_t len,
                                                          uint32_t* part) {
  __shared__ uint32_t sw[32];
  uint32_t t = 0;
  const int64_t base = (int64_t)blockIdx.x * kScanChunk;
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    int64_t j = base + (int64_t)i * kScanBlock + threadIdx.x;
    if (j < len) t += in[j];
  }
  uint32_t tot;
  block_exclusive_scan(t, sw, &tot);
  if (threadIdx.x == 0) part[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(kScanBlock) scan_parts(uint32_t* part, int64_t nparts) {
  __shared__ uint32_t sw[32];
  uint32_t carry = 0;
  for (int64_t b0 = 0; b0 < nparts; b0 += kScanBlock) {
    const int64_t j = b0 + threadIdx.x;
    uint32_t v = j < nparts ? part[j] : 0;
    uint32_t tot;
    uint32_t ex = block_exclusive_scan(v, sw, &tot);
    if (j < nparts) part[j] = carry + ex;
    carry += tot;
  }
}

__global__ void __launch_bounds__(kScanBlock) scan_apply(uint32_t* data, int64_t len,
                                                         const uint32_t* part) {
  __shared__ uint32_t sw[32];
  const int64_t base = (int64_t)blockIdx.x * kScanChunk;
  // blocked arrangement: thread t owns kScanItems consecutive entries
  uint32_t v[kScanItems];
  uint32_t t = 0;
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    int64_t j = base + (int64_t)threadIdx.x * kScanItems + i;
    v[i] = j < len ? data[j] : 0;
    t += v[i];
  }
  uint32_t ex = block_exclusive_scan(t, sw, nullptr) + part[blockIdx.x];
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    int64_t j = base + (int64_t)threadIdx.x * kScanItems + i;
    if (j < len) data[j] = ex;
    ex += v[i];
  }
}

template <bool kFirst>
__global__ void __launch_bounds__(SORT_THREADS) radix_downsweep(KeySrc s, int64_t n, int shift,
                                                                int n_tiles,
                                                                const uint32_t* __restrict__ hist,
                                                                int32_t* __restrict__ keys_out,
                                                                int32_t* __restrict__ vals_out) {
  constexpr int NW = SORT_THREADS / 32;
  constexpr int PER_WARP = SORT_TILE / NW;  // 512 consecutive keys per warp
  __shared__ uint32_t cnt[NW][RADIX_BINS + 1];
  __shared__ uint32_t tdo[RADIX_BINS];      // tile-local exclusive digit offsets
  __shared__ uint32_t gofs[RADIX_BINS];     // global base of (digit, this tile)
  __shared__ uint32_t sw[32];
  __shared__ int32_t sk[SORT_TILE];
  __shared__ int32_t sv[SORT_TILE];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < NW * (RADIX_BINS + 1); i += SORT_THREADS) (&cnt[0][0])[i] = 0;
  __syncthreads();

  const int64_t base = (int64_t)blockIdx.x * SORT_TILE + (int64_t)warp * PER_WARP;
  const unsigned lt_mask = (1u << lane) - 1u;
  int32_t key[SORT_ITEMS], val[SORT_ITEMS];
  uint32_t rank[SORT_ITEMS];
  int dig[SORT_ITEMS];
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    const int64_t j = base + r * 32 + lane;
    int d = RADIX_BINS;  // keys past the end use an extra bin and are never written
    key[r] = 0;
    val[r] = 0;
    if (j < n) {
      load_key<kFirst>(s, j, key[r], val[r]);
      d = (key[r] >> shift) & (RADIX_BINS - 1);
    }
    dig[r] = d;
    const unsigned peers = __match_any_sync(0xffffffffu, d);
    const uint32_t before = cnt[warp][d];
    rank[r] = before + __popc(peers & lt_mask);
    __syncwarp();
    if (lane == __ffs(peers) - 1) cnt[warp][d] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per digit: exclusive prefix over warps, tile total, tile-local digit offsets
  {
    const int d = threadIdx.x;  // SORT_THREADS == RADIX_BINS
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      uint32_t c = cnt[w][d];
      cnt[w][d] = run;
      run += c;
    }
    uint32_t ex = block_exclusive_scan(run, sw, nullptr);
    tdo[d] = ex;
    gofs[d] = hist[(size_t)d * n_tiles + blockIdx.x];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    if (dig[r] < RADIX_BINS) {
      const uint32_t lp = tdo[dig[r]] + cnt[warp][dig[r]] + rank[r];
      sk[lp] = key[r];
      sv[lp] = val[r];
    }
  }
  __syncthreads();
  const int64_t tile0 = (int64_t)blockIdx.x * SORT_TILE;
  const int valid = (int)((n - tile0) < SORT_TILE ? (n - tile0) : SORT_TILE);
  for (int j = threadIdx.x; j < valid; j += SORT_THREADS) {
    const int32_t k = sk[j];
    const int d = (k >> shift) & (RADIX_BINS - 1);
    const int64_t g = (int64_t)gofs[d] + (j - (int64_t)tdo[d]);
    keys_out[g] = k;
    vals_out[g] = sv[j];
  }
}

fkm_status device_scan(uint32_t* data, int64_t len, uint32_t* part, cudaStream_t st) {
  const int64_t nparts = ceil_div(len, kScanChunk);
  scan_reduce<<<(unsigned)nparts, kScanBlock, 0, st>>>(data, len, part);
  scan_parts<<<1, kScanBlock, 0, st>>>(part, nparts);
  scan_apply<<<(unsigned)nparts, kScanBlock, 0, st>>>(data, len, part);
  note_launch(3);
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

}  // namespace

static_assert(SORT_THREADS == RADIX_BINS, "downsweep maps one thread per digit");

size_t argsort_scratch_words(int64_t n) {
  const int64_t tiles = ceil_div(n, SORT_TILE);
  return (size_t)ceil_div(tiles * RADIX_BINS, kScanChunk) + 1;
}

// Sorts a.n keys formed from a.ids; leaves sorted keys / values in
// a.keys_out / a.vals_out (which alias keys0/vals0 or keys1/vals1).
fkm_status launch_argsort_ids(SortArgs& a, cudaStream_t st) {
  if (a.n == 0) {
    a.keys_out = a.keys0;
    a.vals_out = a.vals0;
    return FKM_OK;
  }
  const int n_tiles = (int)ceil_div(a.n, SORT_TILE);
  const int passes = (a.key_bits + RADIX_BITS - 1) / RADIX_BITS;
  const int64_t hlen = (int64_t)n_tiles * RADIX_BINS;
  KeySrc s;
  s.ids = a.ids;
  s.N = a.N;
  s.K = a.K;
  s.sentinel = (int)((a.n / a.N) * a.K);
  s.status = a.status;
  int32_t* kout[2] = {a.keys0, a.keys1};
  int32_t* vout[2] = {a.vals0, a.vals1};
  for (int p = 0; p < (passes > 0 ? passes : 1); ++p) {
    const int shift = p * RADIX_BITS;
    if (p == 0) {
      s.keys = nullptr;
      s.vals = nullptr;
      radix_upsweep<true><<<n_tiles, SORT_THREADS, 0, st>>>(s, a.n, shift, n_tiles, a.hist);
      FKM_TRY(device_scan(a.hist, hlen, a.hist_part, st));
      radix_downsweep<true><<<n_tiles, SORT_THREADS, 0, st>>>(s, a.n, shift, n_tiles, a.hist,
                                                              kout[0], vout[0]);
    } else {
      s.keys = kout[(p - 1) & 1];
      s.vals = vout[(p - 1) & 1];
      radix_upsweep<false><<<n_tiles, SORT_THREADS, 0, st>>>(s, a.n, shift, n_tiles, a.hist);
      FKM_TRY(device_scan(a.hist, hlen, a.hist_part, st));
      radix_downsweep<false><<<n_tiles, SORT_THREADS, 0, st>>>(s, a.n, shift, n_tiles, a.hist,
                                                               kout[p & 1], vout[p & 1]);
    }
    FKM_CUDA_TRY(cudaGetLastError());
    note_launch(2);
  }
  const int last = (passes > 0 ? passes : 1) - 1;
  a.keys_out = kout[last & 1];
  a.vals_out = vout[last & 1];
  return FKM_OK;
}

}  // namespace fkm
