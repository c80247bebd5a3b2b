// Self-test of the bounded device waits every pipelined kernel uses.
//
// The paper has no counterpart: this checks the library's failure path. A
// one-thread kernel waits, with the same bounded mbarrier wait as the
// decode and encode kernels, on a barrier that nothing ever arrives at. The
// wait gives up after the given time, the kernel sets the device status bit
// LLA_DEVICE_WAIT_TIMEOUT and returns, and the context stays usable. No
// fault, trap or unbounded loop is involved.
#include "common.cuh"
#include "internal.h"

namespace lla {
namespace {

__global__ void k_selftest_wait(unsigned long long timeout_ns, unsigned int* status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_mbar_init();
  // nothing arrives: phase 0 never completes
  if (!mbar_wait(b, 0u, timeout_ns)) report_status(status, kStatusWaitTimeout);
}

}  // namespace

lla_status run_selftest_wait(unsigned int timeout_us, cudaStream_t stream) {
  k_selftest_wait<<<1, 1, 0, stream>>>((unsigned long long)timeout_us * 1000ull, status_word());
  return check_cuda(cudaGetLastError(), "launch k_selftest_wait");
}

}  // namespace lla
