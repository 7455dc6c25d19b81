// Self-test of the bounded pipeline wait: one CTA waits on an mbarrier through the same helper
// (mbar_wait_limit) that every TMA / tcgen05 pipeline of the library waits with.  When nothing
// arrives on the barrier the wait gives up after the given limit, the kernel records
// kErrTimeoutSelftest in its device error word and returns, exactly the path a stalled pipeline
// takes, so the host-side error reporting can be checked without stalling a real kernel.  No TMA,
// no tensor memory: nothing is in flight when the wait gives up.
#include <cuda_runtime.h>

#include "../../include/fluxdit.h"
#include "common.cuh"
#include "fluxdit_internal.h"
#include "runner.h"

namespace fdit {

__device__ int g_selftest_error;

__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns, int arrive) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (arrive && threadIdx.x == 0) mbar_arrive(&bar);     // completes phase 0
  const bool ok = mbar_wait_limit(&bar, 0, &abort_flag, limit_ns);
  if (!ok && threadIdx.x == 0) atomicCAS(&g_selftest_error, 0, static_cast<int>(kErrTimeoutSelftest));
}

int selftest_read_device_error(cudaStream_t stream) {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_selftest_error, sizeof(int), 0, cudaMemcpyDeviceToHost, stream) !=
      cudaSuccess)
    return -1;
  cudaMemcpyToSymbolAsync(g_selftest_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
  cudaStreamSynchronize(stream);
  return v;
}

}  // namespace fdit

using namespace fdit;

extern "C" {

int flux_selftest_bounded_wait(unsigned long long limit_ns, int arrive, void* stream) {
  if (limit_ns == 0 || limit_ns > kWaitTimeoutNs)
    return fail(FLUX_EINVAL, "limit_ns %llu outside (0, %llu]", limit_ns,
                static_cast<unsigned long long>(kWaitTimeoutNs));
  if (arrive != 0 && arrive != 1) return fail(FLUX_EINVAL, "arrive must be 0 or 1");
  count_launch();
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, arrive);
  FD_CUDA(cudaGetLastError());
  return FLUX_OK;
}

}  // extern "C"
