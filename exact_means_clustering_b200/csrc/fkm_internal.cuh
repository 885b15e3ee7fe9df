// Internal definitions shared by the library's translation units.
#pragma once
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda_runtime.h>

#include "fkm.h"

namespace fkm {

// Bits of the device status word (workspace slot 0): kernels OR these in.
enum : int {
  ST_TIMEOUT = 1,     // a bounded wait on an mbarrier ran out
  ST_BAD_ID = 2,      // fkm_update got an id outside [0, K)
  ST_INTERNAL = 4,    // an internal consistency check failed
  ST_OOB = 8,         // checked build: a gather / scatter index was out of range
};

// The checked build (FKM_CHECKED): kernels verify the indices they gather and
// scatter with before using them; an out-of-range one sets ST_OOB and the
// access is skipped.  fkm_in_range is always true in the normal build.
#ifdef FKM_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif
__device__ __forceinline__ bool fkm_in_range(int64_t i, int64_t n, int* status) {
  if (!kChecked) return true;
  if (i >= 0 && i < n) return true;
  if (status) atomicOr(status, ST_OOB);
  return false;
}

// Programmatic dependent launch.  The kernels of one Lloyd iteration follow
// each other on one stream; launched with launch_pdl, a kernel's CTAs may be
// scheduled while the kernel before it drains.  Every such kernel calls
// pdl_wait() before it reads or writes global memory: it returns once the
// previous grid has completed and its writes are visible (at once for a
// kernel launched the ordinary way).  pdl_trigger() lets the next kernel be
// scheduled once every CTA of this grid has called it or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Assign tiling: 128 points (TMEM lanes) x 256 centroids (TMEM columns) per
// accumulator; K-chunks of 64 16-bit values (one 128-byte swizzled row).
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int KC = 64;
constexpr int A_CHUNK_BYTES = BM * KC * 2;   // 16 KB
constexpr int B_CHUNK_BYTES = BN * KC * 2;   // 32 KB
constexpr int ASSIGN_THREADS = 320;          // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int TMEM_COLS = 512;               // two 256-column fp32 accumulators

// Update tiling: sorted positions are cut into ranges of SEG_RANGE rows, one
// warp per range.  A segment (run of equal keys) contained in one range is
// finished by that warp; one that spans ranges is summed with fp64 atomics.
constexpr int SEG_RANGE = 256;

// The mean centroid's fixed summation order (center_kernel and the fused
// end-of-iteration kernel): MEAN_CHUNKS contiguous chunks of Kp / MEAN_CHUNKS
// padded rows, MEAN_WAYS strided partials per chunk.  Kp is a multiple of BN,
// so every chunk holds whole rounds of the partials.
constexpr int MEAN_CHUNKS = 8;
constexpr int MEAN_WAYS = 16;
static_assert(BN % (MEAN_CHUNKS * MEAN_WAYS) == 0, "whole rounds of partials per chunk");

// Radix argsort: 8-bit digits, 256 threads x 16 keys per tile.
constexpr int RADIX_BITS = 8;
constexpr int RADIX_BINS = 1 << RADIX_BITS;
constexpr int SORT_THREADS = 256;
constexpr int SORT_ITEMS = 16;
constexpr int SORT_TILE = SORT_THREADS * SORT_ITEMS;

__host__ __device__ inline int elem_bytes(int dtype) { return dtype == FKM_F32 ? 4 : 2; }
__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// thread-local error text (fkm_last_error)
void set_error(const char* fmt, ...);
fkm_status cuda_fail(cudaError_t e, const char* what);

#define FKM_CUDA_TRY(call)                                  \
  do {                                                      \
    cudaError_t e_ = (call);                                \
    if (e_ != cudaSuccess) return ::fkm::cuda_fail(e_, #call); \
  } while (0)

#define FKM_TRY(call)                   \
  do {                                  \
    fkm_status s_ = (call);             \
    if (s_ != FKM_OK) return s_;        \
  } while (0)

// ---------------------------------------------------------------- workspace
// Every buffer the library needs beyond the caller's inputs and outputs lives
// in one caller-provided workspace, carved up by this layout.  Sizes depend on
// B, N, K, D and dtype, never on N*K.
struct Layout;
fkm_status make_layout(int B, int N, int K, int D, int dtype, Layout* L);
struct Layout {
  int B, N, K, D, dtype;
  int Kp;          // K rounded up to BN
  int Dp;          // D rounded up to 8 (the halves of a split row)
  int Dq;          // columns of the quantised centroid / split-point rows
  bool split;      // fp32 input: operands split into bf16 hi + lo
  int m_tiles;     // ceil(N / BM)
  int64_t n_sort;  // B * N keys
  int n_sort_tiles;
  int key_bits;
  bool count_sort;  // one-pass counting sort (K <= CS_MAX_K) instead of LSD radix
  size_t status, mvec, cq, caug, xs, xn, keys0, vals0, keys1, vals1, hist, hist_part,
      segstart, segend, sums64, shiftk, cbuf, scal, cnorm, objk, total;
  int metric;  // FKM_METRIC_*; set by the caller after make_layout (default Euclidean)
};

fkm_status make_layout(int B, int N, int K, int D, int dtype, Layout* L);

template <typename T>
inline T* ws_ptr(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// ---------------------------------------------------------------- launchers
struct AssignArgs {
  int B, N, K, Kp, D, dtype;
  bool split;
  const void* xq;      // bf16/f16 points, or the split [hi|lo] rows for fp32
  int x_row_elems;     // elements per row of xq (D, or 2D when split)
  const void* cq;      // centroid offsets q(c - m) [B, Kp, Dq]
  const void* caug;    // bias slabs [B, Kp, 16]: -n/2 in three 16-bit parts
  const float* xn;     // ||x - m||^2 [B, N] (comparison mode only)
  int32_t* ids;        // [B, N]
  int* status;
  float* dist = nullptr;  // comparison mode: write the [B, N, K] distances here
};
fkm_status launch_assign(const AssignArgs& a, cudaStream_t st);
// Largest D (point tiles streamed with the centroids above 256, fp32: 128).
constexpr int ASSIGN_MAX_D = 4096;
bool assign_smem_plan(int D, bool split, int* nA, int* nS, size_t* smem, bool* stream = nullptr);
fkm_status assign_prepare();

// Per batch mean centroid m [B][D]; q(c - m) rows [B][Kp][Dq] (split rows
// for fp32 are [hi | lo] halves of round_up(D, 8) elements each); and per
// centroid the bias slab [B][Kp][16]: -n/2 as three 16-bit parts, n =
// ||q(c-m)||^2 + 2 m.q(c-m) (zero on padding rows).
constexpr int AUG_SLAB = 16;
// metric: FKM_METRIC_EUCLID (bias slab -n/2), FKM_METRIC_DOT (zero bias) or
// FKM_METRIC_COSINE (rows scaled to unit length first, norms into cnorm [B*K]).
fkm_status launch_prep_centroids(const float* centers, int B, int K, int Kp, int D, int dtype,
                                 float* m, void* cq, void* caug, cudaStream_t st,
                                 int metric = FKM_METRIC_EUCLID, double* cnorm = nullptr);
// The end of a Lloyd iteration in one launch: finalize (counts, new
// centroids from the segment sums, sums64 cleared), the mean centroid m
// (bit for bit launch_prep_centroids'), the next assign's operands and bias
// slabs, and the batch shifts (shift_out [B], optional; max_shift optional,
// zeroed by the caller).  metric: Euclidean, or dot / cosine (the similarity
// finalize; cnorm [B*K] receives the cosine row norms; obj_out [B], optional,
// the objective of the assignment).  For Kp <= 1024, B <= 65535 and D <= 256
// (Euclidean) or D <= 128 (finalize_prep_fits).
bool finalize_prep_fits(int B, int Kp, int D, int metric);
fkm_status launch_finalize_prep(int B, int K, int Kp, int D, int dtype, int range,
                                const int32_t* segstart, const int32_t* segend, double* sums64,
                                const float* prev, float* centers, int32_t* counts, float* m,
                                void* cq, void* caug, double* shift_out, double* max_shift,
                                cudaStream_t st, int metric = FKM_METRIC_EUCLID,
                                double* cnorm = nullptr, double* obj_out = nullptr);
// fp32 points: split rows into xs; xn (optional) = ||x - m[row / N]||^2
// (||x||^2 when m is null).
fkm_status launch_points_prep(const void* x, int64_t rows, int D, int dtype, void* xs, float* xn,
                              cudaStream_t st, const float* m = nullptr, int N = 1);

struct SortArgs {
  const int32_t* ids;  // first-pass keys come from ids: key = (row / N) * K + id
  int N, K;
  int64_t n;           // number of keys
  int key_bits;
  int32_t *keys0, *vals0, *keys1, *vals1;
  uint32_t* hist;      // [RADIX_BINS * tiles]
  uint32_t* hist_part; // scan scratch
  int* status;
  int32_t* keys_out;   // set by the launcher: where the sorted keys / values ended up
  int32_t* vals_out;
};
fkm_status launch_argsort_ids(SortArgs& a, cudaStream_t st);
size_t argsort_scratch_words(int64_t n);

// One-pass counting sort of the same keys for K <= CS_MAX_K: rows of a batch
// are contiguous, so per-batch stable sorts by id concatenate into the stable
// sort by key.  Also writes segstart / segend ([B*K], positions in the sorted
// order; equal for an empty cluster).  hist needs cs_hist_words(B, N, K)
// words, hist_part argsort_scratch_words-style scan scratch for that length.
constexpr int CS_MAX_K = 2048;
int64_t cs_hist_words(int B, int N, int K);
size_t cs_scan_scratch_words(int B, int N, int K);
// ids_valid: every id is known to lie in [0, K) (the assign kernel wrote
// them), which allows the one-launch path for batches of at most SORT_TILE
// points.
fkm_status launch_count_sort_ids(SortArgs& a, int B, int32_t* segstart, int32_t* segend,
                                 cudaStream_t st, bool ids_valid = false);
fkm_status count_sort_prepare();

// Objective of the assignment being summed against c_hat, the centroid the
// assign step measured against: m + q(c - m) for 16-bit points (chat = the
// q(c - m) rows [B][Kp][D], m = the per-batch mean centroid), the fp32
// centroids themselves for fp32 points (chat = [B][K][D], m = nullptr);
// chat_bstride is the batch stride of chat in elements; obj[b] (zeroed by the
// caller) receives sum ||x - c_hat||^2.
struct ObjArgs {
  const void* chat = nullptr;
  int64_t chat_bstride = 0;
  const float* m = nullptr;   // 16-bit chat: c_hat = m[b] + chat (per batch [B][D])
  int K = 1;
  double* obj = nullptr;
};
// atomics (optional): incremented by the number of fp64 element atomics the
// segment sums add into sums64 (D per flush of a run that crosses a range).
// segstart / segend (optional, cleared by clear_seg_bounds first): the
// segment bounds of the sorted keys are written by the same pass.
fkm_status launch_segsum(const void* x, int dtype, int D, const int32_t* skeys,
                         const int32_t* svals, int64_t n, int BK, double* sums64, float* centers,
                         bool accumulate_all, const ObjArgs& oa, cudaStream_t st, int range = 0,
                         unsigned long long* atomics = nullptr, int32_t* segstart = nullptr,
                         int32_t* segend = nullptr, int* status = nullptr);
fkm_status clear_seg_bounds(int BK, int32_t* segstart, int32_t* segend, cudaStream_t st);
// Rows per warp range of the segment sums for n sorted rows: SEG_RANGE for
// large n, fewer (down to 32) when n is small, so a small problem still
// spreads over many warps.  finalize must be given the same value.
int segsum_range_rows(int64_t n);
// Raises the segment-sum kernels' dynamic shared-memory limit once per device
// (outside any stream capture).
fkm_status segsum_prepare();
// Direct objective of a given assignment: obj[b] += sum_i ||x_i - chat_{ids_i}||^2.
fkm_status launch_objective(const void* x, int dtype, int B, int N, int D, const int32_t* ids,
                            const ObjArgs& oa, cudaStream_t st);
// clear_sums: zero sums64 after reading it (the library's own accumulators);
// false leaves a caller's reduced sums untouched.  counts_in64 (fp64 counts,
// the shard partials reduced across GPUs) takes precedence over counts_in.
fkm_status launch_finalize(int B, int K, int D, const int32_t* segstart, const int32_t* segend,
                           const int32_t* counts_in, double* sums64, const float* prev,
                           float* centers, int32_t* counts, double* shiftk, cudaStream_t st,
                           int range = SEG_RANGE, bool clear_sums = true,
                           const double* counts_in64 = nullptr);
fkm_status launch_batch_reduce(int B, int K, const double* shiftk, double* shift_out,
                               double* max_shift, cudaStream_t st);
// dot-product / cosine k-means: new centroids, per-cluster shift and
// objective share (objk [B*K]) from the segment sums; sums64 left zeroed.
// counts_in (out-of-core): accumulated counts, every cluster's sum in sums64
// (segstart / segend unused).
fkm_status launch_finalize_sim(int B, int K, int D, int metric, const int32_t* segstart,
                               const int32_t* segend, double* sums64, const float* prev,
                               float* centers, int32_t* counts, double* shiftk, double* objk,
                               cudaStream_t st, int range, const int32_t* counts_in = nullptr);

fkm_status launch_baseline_argmin(const float* dist, int64_t rows, int K, int32_t* ids,
                                  cudaStream_t st);
fkm_status launch_baseline_update(const void* x, int dtype, const int32_t* ids, int B, int N,
                                  int K, int D, float* sums, int32_t* cnt, const float* prev,
                                  float* centers, int32_t* counts, int* status, cudaStream_t st);

int num_sms();

// Counts kernel launches made by this library (fkm_kernel_launches).
void note_launch(int n = 1);

}  // namespace fkm
