// Self-test of the bounded device waits every tensor-core kernel relies on.
//
// Each wait on an mbarrier (TMA completion, MMA commit, a hand-off between
// warps) gives up after a wall-clock limit read from %globaltimer, and the
// kernel then records MOBA_STATUS_TIMEOUT, winds down and returns, so a lost
// completion never hangs the GPU.  This kernel makes that path run on
// purpose, safely: one mbarrier expects two arrivals and only one is ever
// made, nothing asynchronous (no TMA copy, no MMA) is in flight, and every
// thread waits with the given limit.  The CTA agrees on the outcome, records
// the timeout and exits; the context stays usable.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "moba.h"
#include "tc.cuh"

namespace moba {
namespace {

__global__ void __launch_bounds__(128) wait_selftest_kernel(unsigned long long limit_ns, int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t addr = smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(addr, 2);  // two arrivals complete the phase
    tc::mbar_init_fence();
  }
  __syncthreads();
  if (threadIdx.x == 0) tc::mbar_arrive(addr);  // the second one never comes
  const bool done = tc::mbar_wait(addr, 0, limit_ns);
  const bool all = __syncthreads_and(done);
  if (!all && threadIdx.x == 0) set_status(status, kStatusTimeout);
}

}  // namespace
}  // namespace moba

extern "C" int moba_selftest_bounded_wait(unsigned long long limit_ns, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  if (!workspace || workspace_bytes < 256) return MOBA_EINVAL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOBA_EALIGN;
  if (limit_ns == 0 || limit_ns > 10000000000ull) return MOBA_EINVAL;  // 1 ns .. 10 s
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* status = static_cast<int32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), st) != cudaSuccess) return MOBA_ELAUNCH;
  moba::wait_selftest_kernel<<<1, 128, 0, st>>>(limit_ns, status);
  return cudaGetLastError() == cudaSuccess ? MOBA_OK : MOBA_ELAUNCH;
}
