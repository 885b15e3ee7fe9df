// Self-test of the failure-detection path: a bounded wait that runs out.
//
// Every persistent kernel here (assign, segment sums) waits on mbarriers with
// a bounded wait: after a time limit it gives up, ORs ST_TIMEOUT into the
// workspace's status word and returns, so a lost arrival ends in an error
// status the host reads instead of a hung GPU.  This kernel exercises exactly
// that path without any fault: it waits on an mbarrier that nothing arrives
// on, with a short limit.
#include "fkm_internal.cuh"
#include "ptx_sm100.cuh"

namespace fkm {
namespace {

__global__ void wait_timeout_kernel(int* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);   // expects one arrival; none is ever made
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    ptx::mbar_wait_bounded(&bar, 0, &abort_flag, status, ST_TIMEOUT, timeout_ns);
}

}  // namespace
}  // namespace fkm

using namespace fkm;

extern "C" fkm_status fkm_selftest_wait_timeout(uint64_t timeout_ns, void* ws, size_t ws_bytes,
                                                void* stream) {
  if (!ws || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 15)) {
    set_error("the workspace must be at least 256 bytes and 16-byte aligned");
    return FKM_ERR_INVALID_ARG;
  }
  if (timeout_ns < 1000 || timeout_ns > 1000000000ull) {
    set_error("timeout_ns must lie in [1 us, 1 s]");
    return FKM_ERR_INVALID_ARG;
  }
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int*>(ws),
                                                                       timeout_ns);
  note_launch();
  FKM_CUDA_TRY(cudaGetLastError());
  return FKM_OK;
}
