// fkm_assign_noalloc: the assign step for callers that cannot allocate.
//
// Some callers are not allowed to allocate device memory at the point where
// they need an assignment: code whose device memory is owned by a framework
// allocator that must not be bypassed there, real-time or embedded services
// that reserve all memory up front in fixed pools (a cudaMalloc mid-run can
// stall or fail), plugins handed only their inputs and outputs by a host
// application.  They cannot call cudaMalloc for the workspace that
// fkm_assign expects.
//
// This entry point keeps its scratch (the per-batch mean centroid, the
// centroid offsets rounded to the points' 16-bit type, their bias slabs, and
// a status word) in one file-scope
// device array of FKM_NOALLOC_SCRATCH_BYTES.  Every GPU that loads the library
// holds that array until the process exits.  The host-side name of the array
// is only a stand-in: its device address is fetched with cudaGetSymbolAddress,
// once per device, with that device current, on the first call made on it
// (the address is cached for the life of the process, so a device reset
// while the library is loaded is not supported).  fkm_assign_noalloc_status
// reads and clears the array's status word.
#include <cstring>
#include <mutex>

#include "fkm_internal.cuh"

namespace fkm {
namespace {

constexpr size_t kScratchBytes = FKM_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array for the current device.
fkm_status scratch_for_current_device(void** out) {
  int dev = 0;
  FKM_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) {
    set_error("device index %d out of range", dev);
    return FKM_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_error("cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
      return FKM_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FKM_OK;
}

}  // namespace
}  // namespace fkm

using namespace fkm;

extern "C" fkm_status fkm_assign_noalloc(int B, int N, int K, int D, int dtype, const void* x,
                                         const float* centers, int32_t* ids, void* stream) {
  if (dtype != FKM_BF16 && dtype != FKM_F16) {
    set_error("fkm_assign_noalloc takes bf16 or fp16 points only (fp32 points need scratch "
              "proportional to N)");
    return FKM_ERR_UNSUPPORTED;
  }
  size_t probe = 0;
  FKM_TRY(fkm_workspace_size(B, N, K, D, dtype, &probe));  // shape validation
  const uintptr_t need_align = 15;
  if (!x || !centers || !ids || (reinterpret_cast<uintptr_t>(x) & need_align) ||
      (reinterpret_cast<uintptr_t>(centers) & need_align) ||
      (reinterpret_cast<uintptr_t>(ids) & need_align)) {
    set_error("x, centers and ids must be non-null and 16-byte aligned");
    return FKM_ERR_INVALID_ARG;
  }
  const int Kp = (int)round_up(K, BN);
  const size_t status_bytes = 256;
  const size_t m_bytes = (size_t)round_up((int64_t)B * D * 4, 256);
  const size_t cq_bytes = (size_t)round_up((int64_t)B * Kp * D * 2, 256);
  const size_t aug_bytes = (size_t)round_up((int64_t)B * Kp * AUG_SLAB * 2, 256);
  if (status_bytes + m_bytes + cq_bytes + aug_bytes > kScratchBytes) {
    set_error("B*(4*D + Kp*(2*D + 32)) = %zu bytes exceeds the %zu-byte static scratch of "
              "fkm_assign_noalloc (Kp = K rounded up to 256)",
              m_bytes + cq_bytes + aug_bytes, kScratchBytes - status_bytes);
    return FKM_ERR_UNSUPPORTED;
  }
  void* base = nullptr;
  FKM_TRY(scratch_for_current_device(&base));
  char* p = static_cast<char*>(base);
  int* status = reinterpret_cast<int*>(p);
  float* m = reinterpret_cast<float*>(p + status_bytes);
  void* cq = p + status_bytes + m_bytes;
  void* caug = p + status_bytes + m_bytes + cq_bytes;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word is the only scratch that must start at zero; the rest is
  // fully rewritten by the centroid preparation below
  FKM_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), st));
  FKM_TRY(launch_prep_centroids(centers, B, K, Kp, D, dtype, m, cq, caug, st));
  AssignArgs a;
  a.B = B;
  a.N = N;
  a.K = K;
  a.Kp = Kp;
  a.D = D;
  a.dtype = dtype;
  a.split = false;
  a.xq = x;
  a.x_row_elems = D;
  a.cq = cq;
  a.caug = caug;
  a.xn = nullptr;
  a.ids = ids;
  a.status = status;
  return launch_assign(a, st);
}

extern "C" fkm_status fkm_assign_noalloc_status(void* stream) {
  void* base = nullptr;
  FKM_TRY(scratch_for_current_device(&base));
  int* status = static_cast<int*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int host = 0;
  FKM_CUDA_TRY(cudaMemcpyAsync(&host, status, sizeof(int), cudaMemcpyDeviceToHost, st));
  FKM_CUDA_TRY(cudaStreamSynchronize(st));
  if (host == 0) return FKM_OK;
  FKM_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), st));
  FKM_CUDA_TRY(cudaStreamSynchronize(st));
  if (host & ST_TIMEOUT) {
    set_error("a device-side bounded wait of fkm_assign_noalloc ran out (status 0x%x)", host);
    return FKM_ERR_TIMEOUT;
  }
  set_error("fkm_assign_noalloc device status 0x%x", host);
  return FKM_ERR_INTERNAL;
}
