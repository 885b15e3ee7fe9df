// C ABI of libfkm: argument validation, workspace layout, stream-ordered
// launch sequences, the Lloyd loop and status reporting.  Every step of an
// iteration runs in this library's kernels; there is no fallback path.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "fkm_internal.cuh"

namespace fkm {

static thread_local char g_err[512] = "";

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

fkm_status cuda_fail(cudaError_t e, const char* what) {
  set_error("%s: %s", what, cudaGetErrorString(e));
  return FKM_ERR_CUDA;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

static std::atomic<long long> g_launches{0};
// progress output of the Lloyd loops (fkm_set_verbose)
static std::atomic<int> g_verbose{0};
int verbose_level() { return g_verbose.load(); }
void note_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// ---- stage timing (fkm_profile): CUDA events around each stage of every
// iteration, recorded on the launching stream; inside a stream capture they
// become event-record nodes of the graph (cudaEventRecordExternal)
enum { ST_ASSIGN = 0, ST_SORT = 1, ST_SEGSUM = 2, ST_FINAL = 3, N_STAGES = 4 };
struct Profiler {
  std::mutex mu;
  std::atomic<bool> on{false};
  std::vector<cudaEvent_t> ev;   // 5 per iteration
  int gen = 0;                   // bumped when the event pool changes
  double ms[N_STAGES + 1] = {0};
  long long iters = 0;
};
static Profiler g_prof;

static fkm_status prof_reserve(int iters) {
  const size_t need = (size_t)iters * 5;
  if (g_prof.ev.size() >= need) return FKM_OK;
  while (g_prof.ev.size() < need) {
    cudaEvent_t e;
    FKM_CUDA_TRY(cudaEventCreate(&e));
    g_prof.ev.push_back(e);
  }
  ++g_prof.gen;
  return FKM_OK;
}


// A stage boundary: inside a stream capture the record must become a graph
// node (cudaEventRecordExternal); outside one a plain record is required.
static fkm_status record_stage(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  FKM_CUDA_TRY(cudaStreamIsCapturing(st, &cs));
  if (cs == cudaStreamCaptureStatusActive)
    FKM_CUDA_TRY(cudaEventRecordWithFlags(e, st, cudaEventRecordExternal));
  else
    FKM_CUDA_TRY(cudaEventRecord(e, st));
  return FKM_OK;
}

static void prof_collect(int iters) {
  for (int t = 0; t < iters; ++t) {
    cudaEvent_t* e = &g_prof.ev[(size_t)t * 5];
    float v = 0.0f;
    for (int s = 0; s < N_STAGES; ++s)
      if (cudaEventElapsedTime(&v, e[s], e[s + 1]) == cudaSuccess) g_prof.ms[s] += v;
    if (cudaEventElapsedTime(&v, e[0], e[4]) == cudaSuccess) g_prof.ms[N_STAGES] += v;
  }
  g_prof.iters += iters;
  cudaGetLastError();
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int bits_for(int64_t v) {  // bits needed to hold the value v
  int b = 0;
  while ((int64_t(1) << b) <= v) ++b;
  return b < 1 ? 1 : b;
}

static fkm_status validate_shape(int B, int N, int K, int D, int dtype) {
  if (B < 1 || N < 1 || K < 1 || D < 1) {
    set_error("B, N, K, D must be >= 1 (got %d, %d, %d, %d)", B, N, K, D);
    return FKM_ERR_INVALID_ARG;
  }
  if (dtype != FKM_F32 && dtype != FKM_F16 && dtype != FKM_BF16) {
    set_error("unknown dtype %d", dtype);
    return FKM_ERR_INVALID_ARG;
  }
  const int s = elem_bytes(dtype);
  if ((int64_t)D * s % 16 != 0) {
    set_error("D * sizeof(dtype) = %d is not a multiple of 16 bytes", D * s);
    return FKM_ERR_UNSUPPORTED;
  }
  if (D > ASSIGN_MAX_D) {
    set_error("D = %d exceeds the supported maximum of %d", D, ASSIGN_MAX_D);
    return FKM_ERR_UNSUPPORTED;
  }
  if ((int64_t)B * N >= (int64_t(1) << 31) || (int64_t)B * K >= (int64_t(1) << 31) - 1) {
    set_error("B*N and B*K must stay below 2^31");
    return FKM_ERR_UNSUPPORTED;
  }
  if (!assign_smem_plan(D, dtype == FKM_F32, nullptr, nullptr, nullptr)) {
    set_error("D = %d does not fit the assign kernel's shared memory", D);
    return FKM_ERR_UNSUPPORTED;
  }
  return FKM_OK;
}

fkm_status make_layout(int B, int N, int K, int D, int dtype, Layout* L) {
  FKM_TRY(validate_shape(B, N, K, D, dtype));
  Layout l;
  l.B = B;
  l.N = N;
  l.K = K;
  l.D = D;
  l.dtype = dtype;
  l.split = dtype == FKM_F32;
  l.Kp = (int)round_up(K, BN);
  l.Dp = (int)round_up(D, 8);
  l.Dq = l.split ? 2 * l.Dp : D;
  l.m_tiles = (int)ceil_div(N, BM);
  l.n_sort = (int64_t)B * N;
  l.n_sort_tiles = (int)ceil_div(l.n_sort, SORT_TILE);
  l.key_bits = bits_for((int64_t)B * K);  // includes the sentinel value B*K
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t BN_ = (size_t)B * N, BK = (size_t)B * K;
  l.status = take(256);
  l.mvec = take((size_t)B * D * 4);
  l.cq = take((size_t)B * l.Kp * l.Dq * 2);
  l.caug = take((size_t)B * l.Kp * AUG_SLAB * 2);
  l.xs = take(l.split ? BN_ * l.Dq * 2 : 0);
  l.xn = take(BN_ * 4);
  l.keys0 = take(BN_ * 4);
  l.vals0 = take(BN_ * 4);
  l.keys1 = take(BN_ * 4);
  l.vals1 = take(BN_ * 4);
  l.count_sort = K <= CS_MAX_K;
  {
    size_t hw = (size_t)l.n_sort_tiles * RADIX_BINS, pw = argsort_scratch_words(l.n_sort);
    if (l.count_sort) {
      hw = std::max(hw, (size_t)cs_hist_words(B, N, K));
      pw = std::max(pw, cs_scan_scratch_words(B, N, K));
    }
    l.hist = take(hw * 4);
    l.hist_part = take(pw * 4);
  }
  l.segstart = take(BK * 4);
  l.segend = take(BK * 4);
  l.sums64 = take(BK * D * 8);
  l.shiftk = take(BK * 8);
  l.cbuf = take(2 * BK * D * 4);
  l.scal = take((size_t)B * 8 * 2 + 64);
  l.cnorm = take(BK * 8);
  l.objk = take(BK * 8);
  l.metric = FKM_METRIC_EUCLID;
  l.total = off;
  *L = l;
  return FKM_OK;
}

struct Ws {
  void* base;
  const Layout* L;
  template <typename T>
  T* at(size_t off) const { return ws_ptr<T>(base, off); }
  int* status() const { return at<int>(L->status); }
  double* max_shift() const { return at<double>(L->status + 64); }
  // fp64 atomic additions made by the segment sums (fkm_segsum_stats)
  unsigned long long* atomics() const { return at<unsigned long long>(L->status + 128); }
};

static fkm_status check_ws(const Layout& L, void* ws, size_t ws_bytes) {
  if (!ws || !aligned16(ws)) {
    set_error("workspace pointer is null or not 16-byte aligned");
    return FKM_ERR_INVALID_ARG;
  }
  if (ws_bytes < L.total) {
    set_error("workspace of %zu bytes is smaller than the %zu required", ws_bytes, L.total);
    return FKM_ERR_WORKSPACE_TOO_SMALL;
  }
  return FKM_OK;
}

static fkm_status check_ptr(const void* p, const char* name) {
  if (!p || !aligned16(p)) {
    set_error("%s is null or not 16-byte aligned", name);
    return FKM_ERR_INVALID_ARG;
  }
  return FKM_OK;
}

// ---- the steps of one iteration ----
static fkm_status step_assign(const Ws& w, const void* x, int32_t* ids, cudaStream_t st) {
  const Layout& L = *w.L;
  AssignArgs a;
  a.B = L.B;
  a.N = L.N;
  a.K = L.K;
  a.Kp = L.Kp;
  a.D = L.D;
  a.dtype = L.dtype;
  a.split = L.split;
  a.xq = L.split ? w.at<void>(L.xs) : x;
  a.x_row_elems = L.split ? L.Dq : L.D;
  a.cq = w.at<void>(L.cq);
  a.caug = w.at<void>(L.caug);
  a.xn = nullptr;
  a.ids = ids;
  a.status = w.status();
  return launch_assign(a, st);
}

// The centroid the assign step measured against, as the update's objective
// reads it: q(c) rows in the workspace for 16-bit points, the fp32 centroids
// themselves for fp32 points.
static ObjArgs obj_args(const Ws& w, const float* prev, double* obj) {
  const Layout& L = *w.L;
  ObjArgs o;
  o.K = L.K;
  o.obj = obj;
  if (L.split) {
    o.chat = prev;
    o.chat_bstride = (int64_t)L.K * L.D;
  } else {
    o.chat = w.at<void>(L.cq);
    o.chat_bstride = (int64_t)L.Kp * L.D;
    o.m = w.at<float>(L.mvec);
  }
  return o;
}

// argsort + bounds + segment sums (+ objective) + finalize; prev -> next.
// obj (device [B], zeroed here) receives the objective of ids against prev.
// ids_valid: the ids were written by the assign kernel (all in [0, K)).
// shifts (Lloyd loop): where given, the Euclidean finalize, the next assign's
// operands (requant) and the batch shifts go into one launch, which writes
// shift_out / max_shift and sets *shifts->done; otherwise the caller reduces
// the per-cluster shifts itself.
struct LoopShifts {
  double* shift_out;
  double* max_shift;
  bool done;
};
static fkm_status step_update(const Ws& w, const void* x, const int32_t* ids, const float* prev,
                              float* next, int32_t* counts, bool requant, double* obj,
                              cudaStream_t st, cudaEvent_t* ev = nullptr,
                              bool ids_valid = false, LoopShifts* shifts = nullptr) {
  const Layout& L = *w.L;
  SortArgs s;
  s.ids = ids;
  s.N = L.N;
  s.K = L.K;
  s.n = L.n_sort;
  s.key_bits = L.key_bits;
  s.keys0 = w.at<int32_t>(L.keys0);
  s.vals0 = w.at<int32_t>(L.vals0);
  s.keys1 = w.at<int32_t>(L.keys1);
  s.vals1 = w.at<int32_t>(L.vals1);
  s.hist = w.at<uint32_t>(L.hist);
  s.hist_part = w.at<uint32_t>(L.hist_part);
  s.status = w.status();
  const int BK = L.B * L.K;
  int32_t* segstart = w.at<int32_t>(L.segstart);
  int32_t* segend = w.at<int32_t>(L.segend);
  if (L.count_sort) {
    FKM_TRY(launch_count_sort_ids(s, L.B, segstart, segend, st, ids_valid));
  } else {   // the segment sums write the bounds
    FKM_TRY(launch_argsort_ids(s, st));
    FKM_TRY(clear_seg_bounds(BK, segstart, segend, st));
  }
  if (ev) FKM_TRY(record_stage(ev[2], st));
  const bool euclid = L.metric == FKM_METRIC_EUCLID;
  if (obj && euclid) FKM_CUDA_TRY(cudaMemsetAsync(obj, 0, sizeof(double) * L.B, st));
  const int range = segsum_range_rows(L.n_sort);
  // the Euclidean objective is summed with the rows; the similarity ones come
  // from the cluster sums in the finalize step
  FKM_TRY(launch_segsum(x, L.dtype, L.D, s.keys_out, s.vals_out, L.n_sort, BK,
                        w.at<double>(L.sums64), next, false,
                        obj_args(w, prev, euclid ? obj : nullptr), st, range, w.atomics(),
                        L.count_sort ? nullptr : segstart, L.count_sort ? nullptr : segend,
                        w.status()));
  if (ev) FKM_TRY(record_stage(ev[3], st));
  if (requant && shifts && finalize_prep_fits(L.B, L.Kp, L.D, L.metric)) {
    FKM_TRY(launch_finalize_prep(L.B, L.K, L.Kp, L.D, L.dtype, range, segstart, segend,
                                 w.at<double>(L.sums64), prev, next, counts, w.at<float>(L.mvec),
                                 w.at<void>(L.cq), w.at<void>(L.caug), shifts->shift_out,
                                 shifts->max_shift, st, L.metric, w.at<double>(L.cnorm),
                                 euclid ? nullptr : obj));
    shifts->done = true;
    return FKM_OK;
  }
  if (euclid) {
    FKM_TRY(launch_finalize(L.B, L.K, L.D, segstart, segend, nullptr, w.at<double>(L.sums64),
                            prev, next, counts, w.at<double>(L.shiftk), st, range));
  } else {
    FKM_TRY(launch_finalize_sim(L.B, L.K, L.D, L.metric, segstart, segend,
                                w.at<double>(L.sums64), prev, next, counts,
                                w.at<double>(L.shiftk), w.at<double>(L.objk), st, range));
    if (obj) FKM_TRY(launch_batch_reduce(L.B, L.K, w.at<double>(L.objk), obj, nullptr, st));
  }
  // the next assign's operands: offsets of the new centroids from their mean
  if (requant)
    FKM_TRY(launch_prep_centroids(next, L.B, L.K, L.Kp, L.D, L.dtype, w.at<float>(L.mvec),
                                  w.at<void>(L.cq), w.at<void>(L.caug), st, L.metric,
                                  w.at<double>(L.cnorm)));
  return FKM_OK;
}

static fkm_status read_status(const Ws& w, cudaStream_t st) {
  int host = 0;
  FKM_CUDA_TRY(cudaMemcpyAsync(&host, w.status(), sizeof(int), cudaMemcpyDeviceToHost, st));
  FKM_CUDA_TRY(cudaStreamSynchronize(st));
  if (host == 0) return FKM_OK;
  FKM_CUDA_TRY(cudaMemsetAsync(w.status(), 0, sizeof(int), st));
  if (host & ST_TIMEOUT) {
    set_error("a device-side bounded wait ran out (status 0x%x)", host);
    return FKM_ERR_TIMEOUT;
  }
  if (host & ST_BAD_ID) {
    set_error("an id outside [0, K) was passed to the update (status 0x%x)", host);
    return FKM_ERR_BAD_ID;
  }
  if (host & ST_OOB) {
    set_error("checked build: a kernel met an out-of-range gather or scatter index (status "
              "0x%x)", host);
    return FKM_ERR_INTERNAL;
  }
  set_error("device status 0x%x", host);
  return FKM_ERR_INTERNAL;
}

// ---- CUDA graph of a tol = 0 Lloyd loop, cached for identical calls ----
struct GraphKey {
  int B, N, K, D, dtype, metric, iters;
  const void* x;
  const float* init;
  int32_t* ids;
  float* centers;
  int32_t* counts;
  double* inertia;
  void* ws;
  cudaStream_t st;
  int dev;
  int prof_gen;  // -1 when not profiling
  bool operator==(const GraphKey& o) const { return memcmp(this, &o, sizeof(GraphKey)) == 0; }
};

// A few recent loops stay instantiated (callers that alternate buffers, e.g.
// double-buffered inputs, replay without re-capturing); least recently used
// goes first.
struct GraphEntry {
  GraphKey key;
  cudaGraphExec_t exec;
  long long launches;   // kernels one replay launches
  long long last_use;
};
constexpr size_t kGraphCacheSize = 8;
static std::mutex g_graph_mu;
static std::vector<GraphEntry> g_graphs;
static long long g_graph_clock = 0;

}  // namespace fkm

using namespace fkm;

// Runs iterations [0, iters) of the Lloyd loop on st (no host sync).
// ev_base: profiling events (5 per iteration, indexed by t) or nullptr
static fkm_status lloyd_iterations(const Ws& w, const void* x, int iters, int32_t* ids,
                                   int32_t* counts, double* inertia, double* shift_dev,
                                   bool track_max, int t0, cudaStream_t st,
                                   cudaEvent_t* ev_base) {
  const Layout& L = *w.L;
  float* cA = w.at<float>(L.cbuf);
  float* cB = cA + (size_t)L.B * L.K * L.D;
  for (int t = t0; t < t0 + iters; ++t) {
    float* cur = (t & 1) ? cB : cA;
    float* nxt = (t & 1) ? cA : cB;
    cudaEvent_t* ev = ev_base ? ev_base + (size_t)t * 5 : nullptr;
    if (ev) FKM_TRY(record_stage(ev[0], st));
    FKM_TRY(step_assign(w, x, ids, st));
    if (ev) FKM_TRY(record_stage(ev[1], st));
    if (track_max) FKM_CUDA_TRY(cudaMemsetAsync(w.max_shift(), 0, sizeof(double), st));
    LoopShifts sh{shift_dev, track_max ? w.max_shift() : nullptr, false};
    FKM_TRY(step_update(w, x, ids, cur, nxt, counts, true, inertia, st, ev, true, &sh));
    if (!sh.done)
      FKM_TRY(launch_batch_reduce(L.B, L.K, w.at<double>(L.shiftk), shift_dev,
                                  track_max ? w.max_shift() : nullptr, st));
    if (ev) FKM_TRY(record_stage(ev[4], st));
  }
  return FKM_OK;
}

extern "C" {

const char* fkm_version(void) {
  return kChecked ? "fkm 0.2.0 (sm_100a, checked build)" : "fkm 0.2.0 (sm_100a)";
}

const char* fkm_last_error(void) { return g_err; }

const char* fkm_status_string(fkm_status s) {
  switch (s) {
    case FKM_OK: return "ok";
    case FKM_ERR_INVALID_ARG: return "invalid argument";
    case FKM_ERR_UNSUPPORTED: return "unsupported shape or type";
    case FKM_ERR_CUDA: return "CUDA error";
    case FKM_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case FKM_ERR_TIMEOUT: return "device wait timed out";
    case FKM_ERR_INTERNAL: return "internal error";
    case FKM_ERR_BAD_ID: return "cluster id out of range";
  }
  return "unknown status";
}

fkm_status fkm_workspace_size(int B, int N, int K, int D, int dtype, size_t* bytes) {
  if (!bytes) {
    set_error("bytes is null");
    return FKM_ERR_INVALID_ARG;
  }
  Layout L;
  FKM_TRY(make_layout(B, N, K, D, dtype, &L));
  *bytes = L.total;
  return FKM_OK;
}

static fkm_status check_metric(int metric) {
  if (metric != FKM_METRIC_EUCLID && metric != FKM_METRIC_DOT && metric != FKM_METRIC_COSINE) {
    set_error("metric %d is not one of FKM_METRIC_EUCLID, _DOT, _COSINE", metric);
    return FKM_ERR_INVALID_ARG;
  }
  return FKM_OK;
}

static fkm_status assign_impl(int metric, int B, int N, int K, int D, int dtype, const void* x,
                              const float* centers, int32_t* ids, double* inertia, void* ws,
                              size_t ws_bytes, void* stream) {
  FKM_TRY(check_metric(metric));
  Layout L;
  FKM_TRY(make_layout(B, N, K, D, dtype, &L));
  L.metric = metric;
  FKM_TRY(check_ws(L, ws, ws_bytes));
  FKM_TRY(check_ptr(x, "x"));
  FKM_TRY(check_ptr(centers, "centers"));
  FKM_TRY(check_ptr(ids, "ids"));
  if (inertia) FKM_TRY(check_ptr(inertia, "inertia"));
  if (inertia && B > 65535) {   // the objective kernel runs one grid row per batch
    set_error("fkm_assign's objective needs B <= 65535 (B = %d); pass inertia = NULL or "
              "split the batches", B);
    return FKM_ERR_UNSUPPORTED;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ws w{ws, &L};
  FKM_TRY(launch_prep_centroids(centers, B, K, L.Kp, D, dtype, w.at<float>(L.mvec),
                                w.at<void>(L.cq), w.at<void>(L.caug), st, metric,
                                w.at<double>(L.cnorm)));
  if (L.split)
    FKM_TRY(launch_points_prep(x, L.n_sort, D, dtype, w.at<void>(L.xs), nullptr, st));
  FKM_TRY(step_assign(w, x, ids, st));
  if (inertia) {
    FKM_CUDA_TRY(cudaMemsetAsync(inertia, 0, sizeof(double) * B, st));
    FKM_TRY(launch_objective(x, dtype, B, N, D, ids, obj_args(w, centers, inertia), st));
  }
  return FKM_OK;
}

static fkm_status update_impl(int metric, int B, int N, int K, int D, int dtype, const void* x,
                              const int32_t* ids, const float* prev_centers, float* centers,
                              int32_t* counts, double* shift, double* inertia, void* ws,
                              size_t ws_bytes, void* stream) {
  FKM_TRY(check_metric(metric));
  Layout L;
  FKM_TRY(make_layout(B, N, K, D, dtype, &L));
  L.metric = metric;
  FKM_TRY(check_ws(L, ws, ws_bytes));
  FKM_TRY(check_ptr(x, "x"));
  FKM_TRY(check_ptr(ids, "ids"));
  FKM_TRY(check_ptr(prev_centers, "prev_centers"));
  FKM_TRY(check_ptr(centers, "centers"));
  FKM_TRY(check_ptr(counts, "counts"));
  if (shift) FKM_TRY(check_ptr(shift, "shift"));
  if (inertia) FKM_TRY(check_ptr(inertia, "inertia"));
  if (prev_centers == centers) {
    set_error("centers must not alias prev_centers");
    return FKM_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ws w{ws, &L};
  FKM_CUDA_TRY(cudaMemsetAsync(w.at<double>(L.sums64), 0, (size_t)B * K * D * 8, st));
  if (inertia && !L.split && metric == FKM_METRIC_EUCLID)  // against q(prev), the assign operand
    FKM_TRY(launch_prep_centroids(prev_centers, B, K, L.Kp, D, dtype, w.at<float>(L.mvec),
                                  w.at<void>(L.cq), w.at<void>(L.caug), st));
  FKM_TRY(step_update(w, x, ids, prev_centers, centers, counts, false, inertia, st));
  if (shift) FKM_TRY(launch_batch_reduce(B, K, w.at<double>(L.shiftk), shift, nullptr, st));
  return FKM_OK;
}

static fkm_status lloyd_impl(int metric, int B, int N, int K, int D, int dtype, const void* x,
                             const float* init_centers, int max_iters, float tol, int32_t* ids,
                             float* centers, int32_t* counts, double* inertia, int* n_iter,
                             void* ws, size_t ws_bytes, void* stream) {
  FKM_TRY(check_metric(metric));
  Layout L;
  FKM_TRY(make_layout(B, N, K, D, dtype, &L));
  L.metric = metric;
  FKM_TRY(check_ws(L, ws, ws_bytes));
  FKM_TRY(check_ptr(x, "x"));
  FKM_TRY(check_ptr(init_centers, "init_centers"));
  FKM_TRY(check_ptr(ids, "ids"));
  FKM_TRY(check_ptr(centers, "centers"));
  FKM_TRY(check_ptr(counts, "counts"));
  if (inertia) FKM_TRY(check_ptr(inertia, "inertia"));
  if (!n_iter || max_iters < 1 || !(tol >= 0.0f)) {
    set_error("n_iter must be non-null, max_iters >= 1 and tol >= 0");
    return FKM_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ws w{ws, &L};
  const size_t cbytes = (size_t)B * K * D * sizeof(float);
  float* cA = w.at<float>(L.cbuf);
  float* cB = cA + (size_t)B * K * D;
  double* shift_dev = w.at<double>(L.scal);

  // set-up, outside any graph: status, accumulators, point norms / split
  // operands, the initial centroids and their tensor-core operands
  FKM_CUDA_TRY(cudaMemsetAsync(w.status(), 0, 256, st));
  FKM_CUDA_TRY(cudaMemsetAsync(w.at<double>(L.sums64), 0, (size_t)B * K * D * 8, st));
  FKM_CUDA_TRY(cudaMemcpyAsync(cA, init_centers, cbytes, cudaMemcpyDeviceToDevice, st));
  if (L.split) FKM_TRY(launch_points_prep(x, L.n_sort, D, dtype, w.at<void>(L.xs), nullptr, st));
  FKM_TRY(launch_prep_centroids(cA, B, K, L.Kp, D, dtype, w.at<float>(L.mvec), w.at<void>(L.cq),
                                w.at<void>(L.caug), st, metric, w.at<double>(L.cnorm)));

  // kernel attributes are set here, before any stream capture
  FKM_TRY(assign_prepare());
  FKM_TRY(segsum_prepare());
  FKM_TRY(count_sort_prepare());
  const bool prof = g_prof.on.load();
  std::unique_lock<std::mutex> prof_lock(g_prof.mu, std::defer_lock);
  if (prof) {
    prof_lock.lock();
    FKM_TRY(prof_reserve(max_iters));
  }
  cudaEvent_t* ev_base = prof ? g_prof.ev.data() : nullptr;
  int done = 0;
  // verbose runs take the stepped loop, which reads every iteration's results
  if (tol == 0.0f && g_verbose.load() == 0) {
    // every iteration runs: replay one captured graph of the whole loop
    int dev = 0;
    cudaGetDevice(&dev);
    GraphKey key;
    memset(&key, 0, sizeof(key));
    key.B = B; key.N = N; key.K = K; key.D = D; key.dtype = dtype; key.metric = metric;
    key.iters = max_iters;
    key.x = x; key.init = init_centers; key.ids = ids; key.centers = centers;
    key.counts = counts; key.inertia = inertia; key.ws = ws; key.st = st; key.dev = dev;
    key.prof_gen = prof ? g_prof.gen : -1;
    std::lock_guard<std::mutex> lock(g_graph_mu);
    GraphEntry* hit = nullptr;
    for (auto& ge : g_graphs)
      if (ge.key == key) hit = &ge;
    if (!hit) {
      if (g_graphs.size() >= kGraphCacheSize) {
        size_t lru = 0;
        for (size_t i = 1; i < g_graphs.size(); ++i)
          if (g_graphs[i].last_use < g_graphs[lru].last_use) lru = i;
        cudaGraphExecDestroy(g_graphs[lru].exec);
        g_graphs.erase(g_graphs.begin() + (long)lru);
      }
      cudaGraphExec_t exec = nullptr;
      cudaStream_t cap;
      FKM_CUDA_TRY(cudaStreamCreateWithFlags(&cap, cudaStreamNonBlocking));
      cudaGraph_t g = nullptr;
      const long long l0 = g_launches.load();
      cudaError_t e = cudaStreamBeginCapture(cap, cudaStreamCaptureModeThreadLocal);
      fkm_status s = FKM_OK;
      if (e == cudaSuccess) {
        s = lloyd_iterations(w, x, max_iters, ids, counts, inertia, shift_dev, false, 0, cap,
                             ev_base);
        cudaError_t e2 = cudaStreamEndCapture(cap, &g);
        if (s == FKM_OK && e2 != cudaSuccess) s = cuda_fail(e2, "cudaStreamEndCapture");
      } else {
        s = cuda_fail(e, "cudaStreamBeginCapture");
      }
      if (s == FKM_OK) {
        e = cudaGraphInstantiate(&exec, g, 0);
        if (e != cudaSuccess) {
          exec = nullptr;
          s = cuda_fail(e, "cudaGraphInstantiate");
        }
      }
      if (g) cudaGraphDestroy(g);
      cudaStreamDestroy(cap);
      if (s != FKM_OK) return s;
      g_graphs.push_back(GraphEntry{key, exec, g_launches.load() - l0, 0});
      hit = &g_graphs.back();
    } else {
      note_launch((int)hit->launches);  // the replay launches what the capture counted
    }
    hit->last_use = ++g_graph_clock;
    FKM_CUDA_TRY(cudaGraphLaunch(hit->exec, st));
    done = max_iters;
  } else {
    // verbose: the objective of every iteration's assignment is reported, in
    // the caller's buffer or, without one, in spare workspace doubles
    const bool verbose = g_verbose.load() > 0;
    double* obj = inertia ? inertia : (verbose ? shift_dev + B : nullptr);
    std::vector<double> host_obj(verbose ? (size_t)B : 0);
    for (int t = 0; t < max_iters; ++t) {
      FKM_TRY(lloyd_iterations(w, x, 1, ids, counts, obj, shift_dev, true, t, st, ev_base));
      double mx = 0.0;
      FKM_CUDA_TRY(cudaMemcpyAsync(&mx, w.max_shift(), sizeof(double), cudaMemcpyDeviceToHost, st));
      if (verbose)
        FKM_CUDA_TRY(cudaMemcpyAsync(host_obj.data(), obj, sizeof(double) * B,
                                     cudaMemcpyDeviceToHost, st));
      FKM_CUDA_TRY(cudaStreamSynchronize(st));
      done = t + 1;
      if (verbose) {
        double total = 0.0;
        for (double v : host_obj) total += v;
        fprintf(stderr, "fkm_lloyd: iteration %d/%d  objective %.9g (sum over %d batches)  "
                "max shift %.6g\n", t + 1, max_iters, total, B, mx);
      }
      if (mx < (double)tol) break;
    }
  }
  // the centroids after the last update sit in the buffer that iteration wrote
  float* last = (done & 1) ? cB : cA;
  FKM_CUDA_TRY(cudaMemcpyAsync(centers, last, cbytes, cudaMemcpyDeviceToDevice, st));
  *n_iter = done;
  fkm_status rs = read_status(w, st);
  if (prof) prof_collect(done);
  return rs;
}

fkm_status fkm_assign(int B, int N, int K, int D, int dtype, const void* x, const float* centers,
                      int32_t* ids, double* inertia, void* ws, size_t ws_bytes, void* stream) {
  return assign_impl(FKM_METRIC_EUCLID, B, N, K, D, dtype, x, centers, ids, inertia, ws, ws_bytes,
                     stream);
}

fkm_status fkm_update(int B, int N, int K, int D, int dtype, const void* x, const int32_t* ids,
                      const float* prev_centers, float* centers, int32_t* counts, double* shift,
                      double* inertia, void* ws, size_t ws_bytes, void* stream) {
  return update_impl(FKM_METRIC_EUCLID, B, N, K, D, dtype, x, ids, prev_centers, centers, counts,
                     shift, inertia, ws, ws_bytes, stream);
}

fkm_status fkm_lloyd(int B, int N, int K, int D, int dtype, const void* x,
                     const float* init_centers, int max_iters, float tol, int32_t* ids,
                     float* centers, int32_t* counts, double* inertia, int* n_iter, void* ws,
                     size_t ws_bytes, void* stream) {
  return lloyd_impl(FKM_METRIC_EUCLID, B, N, K, D, dtype, x, init_centers, max_iters, tol, ids,
                    centers, counts, inertia, n_iter, ws, ws_bytes, stream);
}

fkm_status fkm_assign_metric(int B, int N, int K, int D, int dtype, int metric, const void* x,
                             const float* centers, int32_t* ids, void* ws, size_t ws_bytes,
                             void* stream) {
  return assign_impl(metric, B, N, K, D, dtype, x, centers, ids, nullptr, ws, ws_bytes, stream);
}

fkm_status fkm_update_metric(int B, int N, int K, int D, int dtype, int metric, const void* x,
                             const int32_t* ids, const float* prev_centers, float* centers,
                             int32_t* counts, double* shift, double* objective, void* ws,
                             size_t ws_bytes, void* stream) {
  return update_impl(metric, B, N, K, D, dtype, x, ids, prev_centers, centers, counts, shift,
                     objective, ws, ws_bytes, stream);
}

fkm_status fkm_lloyd_metric(int B, int N, int K, int D, int dtype, int metric, const void* x,
                            const float* init_centers, int max_iters, float tol, int32_t* ids,
                            float* centers, int32_t* counts, double* objective, int* n_iter,
                            void* ws, size_t ws_bytes, void* stream) {
  return lloyd_impl(metric, B, N, K, D, dtype, x, init_centers, max_iters, tol, ids, centers,
                    counts, objective, n_iter, ws, ws_bytes, stream);
}

fkm_status fkm_set_verbose(int level) {
  g_verbose = level > 0 ? 1 : 0;
  return FKM_OK;
}

fkm_status fkm_profile(int enable) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  g_prof.on = enable != 0;
  return FKM_OK;
}

fkm_status fkm_profile_read(double* stage_ms, long long* iterations, int reset) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (stage_ms)
    for (int s = 0; s <= N_STAGES; ++s) stage_ms[s] = g_prof.ms[s];
  if (iterations) *iterations = g_prof.iters;
  if (reset) {
    for (int s = 0; s <= N_STAGES; ++s) g_prof.ms[s] = 0.0;
    g_prof.iters = 0;
  }
  return FKM_OK;
}

long long fkm_kernel_launches(void) { return g_launches.load(); }

// Scratch of fkm_argsort: histogram, scan scratch and (counting sort only)
// segment bounds, in 4-byte words.
static void argsort_ws_words(int64_t n, int n_keys, size_t* hist_w, size_t* part_w,
                             size_t* bounds_w) {
  const int64_t m = n > 0 ? n : 1;
  *hist_w = (size_t)ceil_div(m, SORT_TILE) * RADIX_BINS;
  *part_w = argsort_scratch_words(m);
  *bounds_w = 0;
  if (n_keys <= CS_MAX_K) {   // the one-pass counting sort of the Lloyd loop
    *hist_w = std::max(*hist_w, (size_t)cs_hist_words(1, (int)m, n_keys));
    *part_w = std::max(*part_w, cs_scan_scratch_words(1, (int)m, n_keys));
    *bounds_w = 2 * (size_t)n_keys;
  }
}

fkm_status fkm_argsort_workspace_size(int64_t n, int n_keys, size_t* bytes) {
  if (!bytes || n < 0 || n >= (int64_t(1) << 31) || n_keys < 1 || n_keys >= (1 << 30)) {
    set_error("invalid argsort size");
    return FKM_ERR_INVALID_ARG;
  }
  size_t hist_w, part_w, bounds_w;
  argsort_ws_words(n, n_keys, &hist_w, &part_w, &bounds_w);
  size_t off = 256;  // status
  off += 4 * (((size_t)n * 4 + 255) & ~size_t(255));
  off += (hist_w * 4 + 255) & ~size_t(255);
  off += (part_w * 4 + 255) & ~size_t(255);
  off += (bounds_w * 4 + 255) & ~size_t(255);
  *bytes = off;
  return FKM_OK;
}

fkm_status fkm_argsort(const int32_t* keys, int64_t n, int n_keys, int32_t* idx,
                       int32_t* sorted_keys, void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  FKM_TRY(fkm_argsort_workspace_size(n, n_keys, &need));
  if (!ws || !aligned16(ws) || ws_bytes < need) {
    set_error("argsort workspace too small or misaligned");
    return ws_bytes < need ? FKM_ERR_WORKSPACE_TOO_SMALL : FKM_ERR_INVALID_ARG;
  }
  if (n == 0) return FKM_OK;
  FKM_TRY(check_ptr(keys, "keys"));
  FKM_TRY(check_ptr(idx, "idx"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* p = static_cast<char*>(ws);
  const size_t vec = ((size_t)n * 4 + 255) & ~size_t(255);
  size_t hist_w, part_w, bounds_w;
  argsort_ws_words(n, n_keys, &hist_w, &part_w, &bounds_w);
  const size_t hist_b = (hist_w * 4 + 255) & ~size_t(255);
  const size_t part_b = (part_w * 4 + 255) & ~size_t(255);
  SortArgs s;
  s.ids = keys;
  s.N = (int)n;
  s.K = n_keys;
  s.n = n;
  s.key_bits = bits_for(n_keys);
  s.status = reinterpret_cast<int*>(p);
  s.keys0 = reinterpret_cast<int32_t*>(p + 256);
  s.vals0 = reinterpret_cast<int32_t*>(p + 256 + vec);
  s.keys1 = reinterpret_cast<int32_t*>(p + 256 + 2 * vec);
  s.vals1 = reinterpret_cast<int32_t*>(p + 256 + 3 * vec);
  s.hist = reinterpret_cast<uint32_t*>(p + 256 + 4 * vec);
  s.hist_part = reinterpret_cast<uint32_t*>(p + 256 + 4 * vec + hist_b);
  if (bounds_w) {
    int32_t* bounds = reinterpret_cast<int32_t*>(p + 256 + 4 * vec + hist_b + part_b);
    FKM_TRY(launch_count_sort_ids(s, 1, bounds, bounds + n_keys, st));
  } else {
    FKM_TRY(launch_argsort_ids(s, st));
  }
  FKM_CUDA_TRY(cudaMemcpyAsync(idx, s.vals_out, (size_t)n * 4, cudaMemcpyDeviceToDevice, st));
  if (sorted_keys)
    FKM_CUDA_TRY(
        cudaMemcpyAsync(sorted_keys, s.keys_out, (size_t)n * 4, cudaMemcpyDeviceToDevice, st));
  return FKM_OK;
}

fkm_status fkm_baseline_assign(int B, int N, int K, int D, int dtype, const void* x,
                               const float* centers, float* dist, int32_t* ids, void* ws,
                               size_t ws_bytes, void* stream) {
  Layout L;
  FKM_TRY(make_layout(B, N, K, D, dtype, &L));
  FKM_TRY(check_ws(L, ws, ws_bytes));
  FKM_TRY(check_ptr(x, "x"));
  FKM_TRY(check_ptr(centers, "centers"));
  FKM_TRY(check_ptr(dist, "dist"));
  FKM_TRY(check_ptr(ids, "ids"));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ws w{ws, &L};
  FKM_TRY(launch_prep_centroids(centers, B, K, L.Kp, D, dtype, w.at<float>(L.mvec),
                                w.at<void>(L.cq), w.at<void>(L.caug), st));
  FKM_TRY(launch_points_prep(x, L.n_sort, D, dtype, L.split ? w.at<void>(L.xs) : nullptr,
                             w.at<float>(L.xn), st, w.at<float>(L.mvec), N));
  AssignArgs a;
  a.B = B;
  a.N = N;
  a.K = K;
  a.Kp = L.Kp;
  a.D = D;
  a.dtype = dtype;
  a.split = L.split;
  a.xq = L.split ? w.at<void>(L.xs) : x;
  a.x_row_elems = L.split ? L.Dq : D;
  a.cq = w.at<void>(L.cq);
  a.caug = w.at<void>(L.caug);
  a.xn = w.at<float>(L.xn);
  a.ids = ids;
  a.status = w.status();
  a.dist = dist;
  FKM_TRY(launch_assign(a, st));
  return launch_baseline_argmin(dist, L.n_sort, K, ids, st);
}

fkm_status fkm_baseline_update(int B, int N, int K, int D, int dtype, const void* x,
                               const int32_t* ids, const float* prev_centers, float* centers,
                               int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  FKM_TRY(make_layout(B, N, K, D, dtype, &L));
  FKM_TRY(check_ws(L, ws, ws_bytes));
  FKM_TRY(check_ptr(x, "x"));
  FKM_TRY(check_ptr(ids, "ids"));
  FKM_TRY(check_ptr(prev_centers, "prev_centers"));
  FKM_TRY(check_ptr(centers, "centers"));
  FKM_TRY(check_ptr(counts, "counts"));
  Ws w{ws, &L};
  return launch_baseline_update(x, dtype, ids, B, N, K, D, w.at<float>(L.sums64),
                                w.at<int32_t>(L.segstart), prev_centers, centers, counts,
                                w.status(), static_cast<cudaStream_t>(stream));
}

fkm_status fkm_segsum_stats(void* ws, size_t ws_bytes, int64_t n_rows, int reset,
                            unsigned long long* atomics, int* range_rows, void* stream) {
  if (!ws || ws_bytes < 256 || !aligned16(ws) || n_rows < 0) {
    set_error("workspace null, misaligned or smaller than 256 bytes, or n_rows < 0");
    return FKM_ERR_INVALID_ARG;
  }
  if (range_rows) *range_rows = segsum_range_rows(n_rows > 0 ? n_rows : 1);
  if (!atomics && !reset) return FKM_OK;
  Layout L;
  memset(&L, 0, sizeof(L));
  Ws w{ws, &L};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned long long host = 0;
  FKM_CUDA_TRY(cudaMemcpyAsync(&host, w.atomics(), sizeof(host), cudaMemcpyDeviceToHost, st));
  if (reset) FKM_CUDA_TRY(cudaMemsetAsync(w.atomics(), 0, sizeof(host), st));
  FKM_CUDA_TRY(cudaStreamSynchronize(st));
  if (atomics) *atomics = host;
  return FKM_OK;
}

fkm_status fkm_sync_status(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256) {
    set_error("workspace too small");
    return FKM_ERR_INVALID_ARG;
  }
  Layout L;
  memset(&L, 0, sizeof(L));
  L.status = 0;
  Ws w{ws, &L};
  return read_status(w, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
