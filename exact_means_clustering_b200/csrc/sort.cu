// Stable device argsort of the 1-D assignment vector.
//
// Sort-Inverse Update starts by argsorting the assignment vector so equal
// cluster ids form contiguous runs, giving the inverse mapping sorted_idx
// ("Flash-KMeans：快速且内存高效精确K-Means聚类" summary, sections 前置知识 /
// argsort与分段规约 and 方法步骤详情 step (2)).  Keys are key = b*K + id (so
// batches stay apart); values are the row indices b*N + i.
//
// LSD radix sort: as many passes as digits of at most 8 bits need (1 for
// B*K < 256, 2 up to 65536), the key bits split evenly over them.  Per pass:
//   upsweep    tile histograms (4096 keys per 256-thread tile), digit-major
//   scan       exclusive scan of the histogram matrix: global base per
//              (digit, tile)
//   downsweep  stable rank of every key inside its tile (warp multisplit:
//              the lanes holding the same digit found with one ballot per
//              digit bit), keys and values staged in shared memory in sorted
//              order, then written out in contiguous runs per digit.
// The first pass forms the keys from the ids on the fly and validates them:
// an id outside [0, K) sets ST_BAD_ID and gets the sentinel key B*K, which
// sorts after every real key.
//
// For K <= CS_MAX_K the Lloyd loop uses a one-pass counting sort instead.
// The rows of batch b are contiguous, so the stable sort by b*K + id is the
// concatenation of per-batch stable sorts by id: tiles of SORT_TILE rows that
// never straddle a batch count their ids into K bins (plus one bin for
// rejected ids), one exclusive scan over the bins in (batch, id, tile) order
// gives every (id, tile) its output base, and a scatter pass ranks the keys
// stably inside their tile.  The scanned bins are also the segment bounds of
// every cluster, so no separate bounds pass is needed.
#include "fkm_internal.cuh"

namespace fkm {
namespace {

// Lanes of the warp whose value equals this lane's, for values in
// [0, 2^nbits): one ballot per bit, keeping the lanes that agree on it.  The
// hardware match instruction gives the same mask, but its cost grows with
// the number of distinct values in the warp, and with ~32 distinct cluster
// ids per warp it saturated its pipe in the sort kernels.
__device__ __forceinline__ unsigned warp_peers(unsigned v, int nbits) {
  unsigned m = 0xffffffffu;
  for (int i = 0; i < nbits; ++i) {
    const unsigned bit = (v >> i) & 1u;
    const unsigned bal = __ballot_sync(0xffffffffu, bit);
    m &= bit ? bal : ~bal;
  }
  return m;
}

// Bits needed for the values 0..vmax.
__host__ __device__ __forceinline__ int value_bits(unsigned vmax) {
  int b = 1;
  while (b < 32 && (vmax >> b)) ++b;
  return b;
}

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
    // j < 2^31 (B*N is bounded by validation): a 32-bit division suffices
    const int32_t b = (int32_t)((uint32_t)j / (uint32_t)s.N);
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
                                                              int bits, int n_tiles,
                                                              uint32_t* hist) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  const int nbins = 1 << bits;
  __shared__ uint32_t h[SORT_THREADS / 32][RADIX_BINS];
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (SORT_THREADS / 32) * RADIX_BINS; i += SORT_THREADS)
    (&h[0][0])[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * SORT_TILE;
  // every load of the tile first, so they are in flight together; the
  // shared-memory atomics after them would otherwise keep each load behind
  // the previous item's update
  int digit[SORT_ITEMS];
#pragma unroll
  for (int it = 0; it < SORT_ITEMS; ++it) {
    const int64_t j = base + (int64_t)it * SORT_THREADS + threadIdx.x;
    digit[it] = nbins;  // out of range: matches nothing real
    if (j < n) {
      int32_t key, val;
      load_key<kFirst>(s, j, key, val);
      digit[it] = (key >> shift) & (nbins - 1);
    }
  }
#pragma unroll
  for (int it = 0; it < SORT_ITEMS; ++it)
    if (digit[it] < nbins) atomicAdd(&h[warp][digit[it]], 1u);
  __syncthreads();
  for (int d = threadIdx.x; d < nbins; d += SORT_THREADS) {
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < SORT_THREADS / 32; ++w) t += h[w][d];
    hist[(size_t)d * n_tiles + blockIdx.x] = t;
  }
}

// --- device-wide exclusive scan of uint32: chunk totals, then every chunk scans itself ---
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
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
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

// Chunk i adds the totals of chunks 0..i-1 itself (a block sum over at most
// a few thousand words in L2), so no separate pass scans the chunk totals.
__global__ void __launch_bounds__(kScanBlock) scan_apply(uint32_t* data, int64_t len,
                                                         const uint32_t* part) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  __shared__ uint32_t sw[32];
  uint32_t earlier = 0;
  for (int64_t j = threadIdx.x; j < (int64_t)blockIdx.x; j += kScanBlock) earlier += part[j];
  uint32_t carry;
  block_exclusive_scan(earlier, sw, &carry);
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
  uint32_t ex = block_exclusive_scan(t, sw, nullptr) + carry;
#pragma unroll
  for (int i = 0; i < kScanItems; ++i) {
    int64_t j = base + (int64_t)threadIdx.x * kScanItems + i;
    if (j < len) data[j] = ex;
    ex += v[i];
  }
}

// The downsweep runs DS_THREADS threads of DS_ITEMS keys on the same
// SORT_TILE-key tile as the upsweep: with half the per-thread state of a
// 256-thread block, twice as many warps stay resident to cover the loads.
constexpr int DS_THREADS = 2 * SORT_THREADS;
constexpr int DS_ITEMS = SORT_TILE / DS_THREADS;
static_assert(DS_THREADS >= RADIX_BINS, "one thread per digit in the digit scan");

template <bool kFirst>
__global__ void __launch_bounds__(DS_THREADS, 2) radix_downsweep(KeySrc s, int64_t n, int shift,
                                                              int bits, int n_tiles,
                                                              const uint32_t* __restrict__ hist,
                                                              int32_t* __restrict__ keys_out,
                                                              int32_t* __restrict__ vals_out) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  constexpr int NW = DS_THREADS / 32;
  constexpr int PER_WARP = SORT_TILE / NW;  // 256 consecutive keys per warp
  static_assert(NW * (RADIX_BINS + 1) <= 2 * SORT_TILE, "the counters fit the staging area");
  // the per-warp digit counters are only needed until every key knows its
  // place in the tile, so they share memory with the staged keys and values
  __shared__ int32_t stage[2 * SORT_TILE];
  __shared__ uint32_t tdo[RADIX_BINS];      // tile-local exclusive digit offsets
  __shared__ uint32_t gofs[RADIX_BINS];     // global base of (digit, this tile)
  __shared__ uint32_t sw[32];
  int32_t* sk = stage;
  int32_t* sv = stage + SORT_TILE;
  uint32_t (*cnt)[RADIX_BINS + 1] = reinterpret_cast<uint32_t (*)[RADIX_BINS + 1]>(stage);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbins = 1 << bits;
  for (int i = threadIdx.x; i < NW * (RADIX_BINS + 1); i += DS_THREADS) (&cnt[0][0])[i] = 0;
  // this tile's global base of every digit (the scanned histogram), loaded
  // now so its latency overlaps the key loads and the ranking
  const uint32_t gbase =
      (int)threadIdx.x < nbins ? hist[(size_t)threadIdx.x * n_tiles + blockIdx.x] : 0u;
  __syncthreads();

  const int64_t base = (int64_t)blockIdx.x * SORT_TILE + (int64_t)warp * PER_WARP;
  const unsigned lt_mask = (1u << lane) - 1u;
  int32_t key[DS_ITEMS], val[DS_ITEMS];
  uint32_t dr[DS_ITEMS];   // digit (9 bits) | rank inside the warp's items << 9
  // every load first, so they are in flight together (the ranking below
  // goes through shared memory item by item)
#pragma unroll
  for (int r = 0; r < DS_ITEMS; ++r) {
    const int64_t j = base + r * 32 + lane;
    int d = nbins;  // keys past the end use an extra bin and are never written
    key[r] = 0;
    val[r] = 0;
    if (j < n) {
      load_key<kFirst>(s, j, key[r], val[r]);
      d = (key[r] >> shift) & (nbins - 1);
    }
    dr[r] = (uint32_t)d;
  }
#pragma unroll
  for (int r = 0; r < DS_ITEMS; ++r) {
    const int d = (int)dr[r];
    const unsigned peers = warp_peers((unsigned)d, bits + 1);   // digits 0..nbins
    const uint32_t before = cnt[warp][d];
    dr[r] = (uint32_t)d | ((before + __popc(peers & lt_mask)) << 9);
    __syncwarp();
    if (lane == __ffs(peers) - 1) cnt[warp][d] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per digit (threads 0..255): exclusive prefix over warps, tile total,
  // tile-local digit offsets; the other threads add zeros to the block scan
  {
    const int d = threadIdx.x;
    uint32_t run = 0;
    if (d < nbins) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        uint32_t c = cnt[w][d];
        cnt[w][d] = run;
        run += c;
      }
    }
    uint32_t ex = block_exclusive_scan(run, sw, nullptr);
    if (d < nbins) {
      tdo[d] = ex;
      gofs[d] = gbase;
    }
  }
  __syncthreads();
  // every key's place in the tile (while the counters are still there) ...
#pragma unroll
  for (int r = 0; r < DS_ITEMS; ++r) {
    const int d = (int)(dr[r] & 511u);
    dr[r] = d < nbins ? tdo[d] + cnt[warp][d] + (dr[r] >> 9) : 0xffffffffu;
  }
  __syncthreads();
  // ... then the keys staged there in sorted order
#pragma unroll
  for (int r = 0; r < DS_ITEMS; ++r) {
    if (dr[r] != 0xffffffffu) {
      sk[dr[r]] = key[r];
      sv[dr[r]] = val[r];
    }
  }
  __syncthreads();
  const int64_t tile0 = (int64_t)blockIdx.x * SORT_TILE;
  const int valid = (int)((n - tile0) < SORT_TILE ? (n - tile0) : SORT_TILE);
  for (int j = threadIdx.x; j < valid; j += DS_THREADS) {
    const int32_t k = sk[j];
    const int d = (k >> shift) & (nbins - 1);
    const int64_t g = (int64_t)gofs[d] + (j - (int64_t)tdo[d]);
    if (!fkm_in_range(g, n, s.status)) continue;
    keys_out[g] = k;
    vals_out[g] = sv[j];
  }
}

// ---- one-pass counting sort ----
struct CsArgs {
  const int32_t* ids;
  int B, N, K;
  int tpb;               // tiles per batch
  uint32_t* hist;        // [(b*K + k) * tpb + t], then [B*K*tpb + tile] rejected ids
  int* status;
  int32_t* keys_out;
  int32_t* vals_out;
  int32_t* segstart;
  int32_t* segend;
};

// Tile histogram: bins 0..K-1 are the ids, bin K the rejected ids.
__global__ void __launch_bounds__(SORT_THREADS) cs_hist_kernel(CsArgs a) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  extern __shared__ uint32_t h[];   // K + 1
  const int tg = blockIdx.x, b = tg / a.tpb, t = tg % a.tpb;
  for (int i = threadIdx.x; i <= a.K; i += SORT_THREADS) h[i] = 0;
  __syncthreads();
  const int64_t row0 = (int64_t)b * a.N + (int64_t)t * SORT_TILE;
  const int nrows = (a.N - t * SORT_TILE) < SORT_TILE ? (a.N - t * SORT_TILE) : SORT_TILE;
  int id[SORT_ITEMS];
#pragma unroll
  for (int it = 0; it < SORT_ITEMS; ++it) {
    const int i = it * SORT_THREADS + threadIdx.x;
    id[it] = i < nrows ? a.ids[row0 + i] : -2;
  }
  bool bad = false;
#pragma unroll
  for (int it = 0; it < SORT_ITEMS; ++it) {
    const int i = it * SORT_THREADS + threadIdx.x;
    int bin = a.K + 1;   // past the tile: counted nowhere
    if (i < nrows) {
      if (id[it] < 0 || id[it] >= a.K) {
        bin = a.K;
        bad = true;
      } else {
        bin = id[it];
      }
    }
    if (bin <= a.K) atomicAdd(&h[bin], 1u);
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(a.status, ST_BAD_ID);
  for (int k = threadIdx.x; k < a.K; k += SORT_THREADS)
    a.hist[((int64_t)b * a.K + k) * a.tpb + t] = h[k];
  if (threadIdx.x == 0) a.hist[(int64_t)a.B * a.K * a.tpb + tg] = h[a.K];
}

// Shared memory of the scatter pass, in 32-bit words: the per-warp bin
// counters, which the staged (key, row) pairs of the tile reuse once every
// row knows its place, then the bins' tile starts and their global shifts.
__host__ __device__ __forceinline__ int cs_scatter_stage_words(int K) {
  const int counters = (SORT_THREADS / 32) * (K + 1);
  return counters > 2 * SORT_TILE ? counters : 2 * SORT_TILE;
}
__host__ __device__ __forceinline__ size_t cs_scatter_smem_bytes(int K) {
  return ((size_t)cs_scatter_stage_words(K) + 2 * (size_t)(K + 1)) * 4;
}

// Stable scatter of one tile: warp w ranks rows [512 w, 512 w + 512) of the
// tile in order with per-warp bin counters (warp multisplit).  The counters
// become offsets inside each bin (earlier warps first), a block scan of the
// bin totals gives each bin's start in the tile's sorted order, and every row
// stages its key and index at its sorted place in shared memory.  The staged
// tile is then written out in order, so the rows of a bin (consecutive in the
// output) leave as contiguous runs instead of one scattered word per row.
// Tile 0 of each batch also writes that batch's segment bounds.  Four blocks
// per SM keep a 32-batch grid of 16 tiles each (512 blocks) in one wave.
__global__ void __launch_bounds__(SORT_THREADS, 4) cs_scatter_kernel(CsArgs a) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  constexpr int NW = SORT_THREADS / 32;
  constexpr int PER_WARP = SORT_TILE / NW;
  extern __shared__ uint32_t smem[];
  __shared__ uint32_t sw[32];
  const int KB = a.K + 1;
  uint32_t* cnt = smem;                                   // NW * KB, then the staged tile
  uint32_t* start = smem + cs_scatter_stage_words(a.K);   // KB: bin start in the tile
  int32_t* shift = reinterpret_cast<int32_t*>(start + KB);  // KB: global - tile position
  const int tg = blockIdx.x, b = tg / a.tpb, t = tg % a.tpb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < NW * KB; i += SORT_THREADS) cnt[i] = 0;
  const int64_t row0 = (int64_t)b * a.N + (int64_t)t * SORT_TILE;
  const int nrows = (a.N - t * SORT_TILE) < SORT_TILE ? (a.N - t * SORT_TILE) : SORT_TILE;
  int bin[SORT_ITEMS];
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    const int i = warp * PER_WARP + r * 32 + lane;
    bin[r] = a.K + 1;
    if (i < nrows) {
      const int id = a.ids[row0 + i];
      bin[r] = (id < 0 || id >= a.K) ? a.K : id;
    }
  }
  // thread t owns bins [t*kpt, (t+1)*kpt) in the bin scan below; their global
  // bases (the scanned histogram) are loaded together with the ids and parked
  // in `shift`, so the latency of these scattered words is paid once
  const int kpt = (KB + SORT_THREADS - 1) / SORT_THREADS;
  const int k0 = threadIdx.x * kpt;
  {
    constexpr int KPT_MAX = (CS_MAX_K + 1 + SORT_THREADS - 1) / SORT_THREADS;
    uint32_t gv[KPT_MAX];   // every load issued before the first store waits
#pragma unroll
    for (int i = 0; i < KPT_MAX; ++i) {
      const int k = k0 + i;
      gv[i] = 0;
      if (i < kpt && k < KB)
        gv[i] = k < a.K ? a.hist[((int64_t)b * a.K + k) * a.tpb + t]
                        : a.hist[(int64_t)a.B * a.K * a.tpb + tg];
    }
#pragma unroll
    for (int i = 0; i < KPT_MAX; ++i)
      if (i < kpt && k0 + i < KB) shift[k0 + i] = (int32_t)gv[i];
  }
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
  const int nbits = value_bits((unsigned)a.K + 1);   // bins 0..K+1
  uint32_t* wc = cnt + warp * KB;
  // after ranking, bin[r] holds the bin in its low 16 bits and the row's rank
  // among the warp's rows of that bin (< SORT_TILE) in its high 16 bits
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    const unsigned peers = warp_peers((unsigned)bin[r], nbits);
    uint32_t before = 0;
    if (bin[r] <= a.K) before = wc[bin[r]];
    const uint32_t rank = before + __popc(peers & lt_mask);
    __syncwarp();
    if (bin[r] <= a.K && lane == __ffs(peers) - 1) wc[bin[r]] = before + __popc(peers);
    __syncwarp();
    bin[r] |= (int)(rank << 16);
  }
  __syncthreads();
  // per bin: earlier warps' counts become offsets inside the bin; thread t
  // owns bins [t*kpt, (t+1)*kpt) and scans their totals across the block
  uint32_t local = 0;
  for (int k = k0; k < k0 + kpt && k < KB; ++k) {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const uint32_t c = cnt[w * KB + k];
      cnt[w * KB + k] = run;
      run += c;
    }
    start[k] = run;
    local += run;
  }
  uint32_t pos = block_exclusive_scan(local, sw, nullptr);
  for (int k = k0; k < k0 + kpt && k < KB; ++k) {
    const uint32_t n = start[k];
    start[k] = pos;
    shift[k] -= (int32_t)pos;   // global base - tile position
    pos += n;
  }
  __syncthreads();
  // each row's place in the tile's sorted order (bin[r] becomes it)
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    const int k = bin[r] & 0xffff;
    bin[r] = k <= a.K ? (int)(start[k] + wc[k] + ((uint32_t)bin[r] >> 16)) | (k << 16) : -1;
  }
  __syncthreads();   // the counters are dead: the staged tile takes their place
  int32_t* sk = reinterpret_cast<int32_t*>(smem);
  int32_t* sv = sk + SORT_TILE;
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    if (bin[r] >= 0) {
      const int lp = bin[r] & 0xffff;
      sk[lp] = bin[r] >> 16;
      sv[lp] = (int32_t)(row0 + warp * PER_WARP + r * 32 + lane);
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < nrows; j += SORT_THREADS) {
    const int k = sk[j];
    const int64_t g = (int64_t)j + shift[k];
    if (!fkm_in_range(g, (int64_t)a.B * a.N, a.status)) continue;
    a.keys_out[g] = k < a.K ? b * a.K + k : a.B * a.K;
    a.vals_out[g] = sv[j];
  }
  if (t == 0) {
    for (int k = threadIdx.x; k < a.K; k += SORT_THREADS) {
      const int64_t key = (int64_t)b * a.K + k;
      a.segstart[key] = (int32_t)a.hist[key * a.tpb];
      a.segend[key] = (int32_t)a.hist[(key + 1) * a.tpb];
    }
  }
}

// Small batches (N <= SORT_TILE, every id valid): one block per batch does the
// whole counting sort of that batch -- stable per-warp ranking as in the
// scatter pass, the bin totals scanned inside the block, then the scatter --
// and writes the batch's segment bounds.  Batch b's keys occupy positions
// [b*N, (b+1)*N).  One launch instead of five.
__global__ void __launch_bounds__(SORT_THREADS) cs_single_tile_kernel(CsArgs a) {
  pdl_wait();   // the previous kernel of the stream has completed
  pdl_trigger();
  constexpr int NW = SORT_THREADS / 32;
  constexpr int PER_WARP = SORT_TILE / NW;
  extern __shared__ uint32_t cnt[];   // NW * (K + 1) per-warp counters, then K + 1 bin starts
  __shared__ uint32_t sw[32];
  const int KB = a.K + 1;
  uint32_t* start = cnt + NW * KB;
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < NW * KB; i += SORT_THREADS) cnt[i] = 0;
  const int64_t row0 = (int64_t)b * a.N;
  int bin[SORT_ITEMS];
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    const int i = warp * PER_WARP + r * 32 + lane;
    bin[r] = a.K + 1;
    if (i < a.N) {
      const int id = a.ids[row0 + i];
      bin[r] = (id < 0 || id >= a.K) ? a.K : id;   // cannot happen for valid ids
    }
  }
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
  const int nbits = value_bits((unsigned)a.K + 1);   // bins 0..K+1
  uint32_t* wc = cnt + warp * KB;
  uint32_t rank[SORT_ITEMS];
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    const unsigned peers = warp_peers((unsigned)bin[r], nbits);
    uint32_t before = 0;
    if (bin[r] <= a.K) before = wc[bin[r]];
    rank[r] = before + __popc(peers & lt_mask);
    __syncwarp();
    if (bin[r] <= a.K && lane == __ffs(peers) - 1) wc[bin[r]] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // per bin: earlier warps' counts become offsets; the bin total is kept
  for (int k = threadIdx.x; k < KB; k += SORT_THREADS) {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const uint32_t c = cnt[w * KB + k];
      cnt[w * KB + k] = run;
      run += c;
    }
    start[k] = run;
  }
  __syncthreads();
  // exclusive scan of the bin totals: thread t owns bins [t*kpt, (t+1)*kpt)
  const int kpt = (KB + SORT_THREADS - 1) / SORT_THREADS;
  const int k0 = threadIdx.x * kpt;
  uint32_t local = 0;
  for (int k = k0; k < k0 + kpt && k < KB; ++k) local += start[k];
  uint32_t run = (uint32_t)row0 + block_exclusive_scan(local, sw, nullptr);
  for (int k = k0; k < k0 + kpt && k < KB; ++k) {
    const uint32_t n = start[k];
    start[k] = run;
    if (k < a.K) {
      a.segstart[(int64_t)b * a.K + k] = (int32_t)run;
      a.segend[(int64_t)b * a.K + k] = (int32_t)(run + n);
    }
    run += n;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < SORT_ITEMS; ++r) {
    if (bin[r] < a.K) {
      const uint32_t pos = start[bin[r]] + wc[bin[r]] + rank[r];
      if (!fkm_in_range(pos, (int64_t)a.B * a.N, a.status)) continue;
      a.keys_out[pos] = b * a.K + bin[r];
      a.vals_out[pos] = (int32_t)(row0 + warp * PER_WARP + r * 32 + lane);
    }
  }
}

fkm_status device_scan(uint32_t* data, int64_t len, uint32_t* part, cudaStream_t st) {
  const int64_t nparts = ceil_div(len, kScanChunk);
  FKM_CUDA_TRY(launch_pdl(scan_reduce, dim3((unsigned)nparts), dim3(kScanBlock), 0, st,
                          data, len, part));
  FKM_CUDA_TRY(launch_pdl(scan_apply, dim3((unsigned)nparts), dim3(kScanBlock), 0, st,
                          data, len, part));
  note_launch(2);
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}

}  // namespace

static_assert(SORT_THREADS == RADIX_BINS, "downsweep maps one thread per digit");

size_t argsort_scratch_words(int64_t n) {
  const int64_t tiles = ceil_div(n, SORT_TILE);
  return (size_t)ceil_div(tiles * RADIX_BINS, kScanChunk) + 1;
}

int64_t cs_hist_words(int B, int N, int K) {
  const int64_t tpb = ceil_div(N, SORT_TILE);
  return (int64_t)B * K * tpb + (int64_t)B * tpb;
}

size_t cs_scan_scratch_words(int B, int N, int K) {
  return (size_t)ceil_div(cs_hist_words(B, N, K), kScanChunk) + 1;
}

fkm_status count_sort_prepare() {
  static bool done[64] = {false};
  int dev = 0;
  FKM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && done[dev]) return FKM_OK;
  const int b = (int)cs_scatter_smem_bytes(CS_MAX_K);
  FKM_CUDA_TRY(cudaFuncSetAttribute(cs_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, b));
  const int b1 = (SORT_THREADS / 32 + 1) * (CS_MAX_K + 1) * 4;
  FKM_CUDA_TRY(
      cudaFuncSetAttribute(cs_single_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, b1));
  if (dev >= 0 && dev < 64) done[dev] = true;
  return FKM_OK;
}

fkm_status launch_count_sort_ids(SortArgs& s, int B, int32_t* segstart, int32_t* segend,
                                 cudaStream_t st, bool ids_valid) {
  if (s.K > CS_MAX_K || s.n != (int64_t)B * s.N) {
    set_error("count sort: K = %d exceeds %d or n != B*N", s.K, CS_MAX_K);
    return FKM_ERR_INTERNAL;
  }
  FKM_TRY(count_sort_prepare());
  CsArgs a;
  a.ids = s.ids;
  a.B = B;
  a.N = s.N;
  a.K = s.K;
  a.tpb = (int)ceil_div(s.N, SORT_TILE);
  a.hist = s.hist;
  a.status = s.status;
  a.keys_out = s.keys0;
  a.vals_out = s.vals0;
  a.segstart = segstart;
  a.segend = segend;
  s.keys_out = s.keys0;
  s.vals_out = s.vals0;
  if (s.n == 0) return FKM_OK;
  const unsigned tiles = (unsigned)((int64_t)B * a.tpb);
  if (ids_valid && a.tpb == 1) {
    const size_t smem = (size_t)(SORT_THREADS / 32 + 1) * (a.K + 1) * 4;
    FKM_CUDA_TRY(launch_pdl(cs_single_tile_kernel, dim3((unsigned)B), dim3(SORT_THREADS), smem,
                            st, a));
    note_launch();
    FKM_CUDA_TRY(cudaGetLastError());
    return FKM_OK;
  }
  FKM_CUDA_TRY(launch_pdl(cs_hist_kernel, dim3(tiles), dim3(SORT_THREADS), (a.K + 1) * 4, st, a));
  FKM_TRY(device_scan(a.hist, cs_hist_words(B, s.N, s.K), s.hist_part, st));
  FKM_CUDA_TRY(launch_pdl(cs_scatter_kernel, dim3(tiles), dim3(SORT_THREADS),
                          cs_scatter_smem_bytes(a.K), st, a));
  note_launch(2);
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
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
  // the key bits split evenly over the passes (12-bit keys: two 6-bit
  // digits), so no pass ranks more bins than it needs, and the scatter's runs
  // per digit stay long in every pass
  const int bits = passes > 0 ? (a.key_bits + passes - 1) / passes : 1;
  const int64_t hlen = (int64_t)n_tiles << bits;
  KeySrc s;
  s.ids = a.ids;
  s.N = a.N;
  s.K = a.K;
  s.sentinel = (int)((a.n / a.N) * a.K);
  s.status = a.status;
  int32_t* kout[2] = {a.keys0, a.keys1};
  int32_t* vout[2] = {a.vals0, a.vals1};
  for (int p = 0; p < (passes > 0 ? passes : 1); ++p) {
    const int shift = p * bits;
    if (p == 0) {
      s.keys = nullptr;
      s.vals = nullptr;
      FKM_CUDA_TRY(launch_pdl((radix_upsweep<true>), dim3(n_tiles), dim3(SORT_THREADS), 0, st,
                              s, a.n, shift, bits, n_tiles, a.hist));
      FKM_TRY(device_scan(a.hist, hlen, a.hist_part, st));
      FKM_CUDA_TRY(launch_pdl((radix_downsweep<true>), dim3(n_tiles), dim3(DS_THREADS), 0, st,
                              s, a.n, shift, bits, n_tiles, a.hist, kout[0], vout[0]));
    } else {
      s.keys = kout[(p - 1) & 1];
      s.vals = vout[(p - 1) & 1];
      FKM_CUDA_TRY(launch_pdl((radix_upsweep<false>), dim3(n_tiles), dim3(SORT_THREADS), 0, st,
                              s, a.n, shift, bits, n_tiles, a.hist));
      FKM_TRY(device_scan(a.hist, hlen, a.hist_part, st));
      FKM_CUDA_TRY(launch_pdl((radix_downsweep<false>), dim3(n_tiles), dim3(DS_THREADS), 0, st,
                              s, a.n, shift, bits, n_tiles, a.hist, kout[p & 1], vout[p & 1]));
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
