// watchdog.cu -- a self-test of the bounded waits that every kernel of the library relies on.
//
// Every mbarrier wait in the kernels gives up after a bounded number of SM cycles, records
// CSA_ERR_TIMEOUT (and the wait's site) in the workspace's status word and lets its CTA unwind, so
// a stalled pipeline is reported instead of hanging the GPU. This kernel runs that same wait
// (mbar_wait) on a phase that nothing completes, with a caller-chosen limit: it must give up,
// record the status and return, leaving the context usable. It moves no data and touches only the
// status word.

#include "csa.h"
#include "kernels.cuh"
#include "ptx.cuh"

namespace csa {

constexpr uint32_t kWatchdogSite = 900;

__global__ void watchdog_kernel(uint32_t* status, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival would complete phase 0; none ever comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, kWatchdogSite, limit);
}

}  // namespace csa

extern "C" int csa_watchdog_selftest(void* ws, size_t ws_bytes, long long limit_cycles, void* stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < csa::kStatusBytes)
    return CSA_ERR_WORKSPACE;
  if (limit_cycles < 1 || limit_cycles > csa::kWaitCycles) return CSA_ERR_INVALID_ARG;
  csa::watchdog_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(ws), limit_cycles);
  return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}
