// Self-test of the device-side wait limit, for tests and health checks of
// failure detection (it has no counterpart in the method). One block waits on
// an mbarrier that nothing will ever arrive on; the wait gives up after the
// same 2 s limit that every wait in the library has, records error 1 in the
// workspace error word and returns, so the context stays usable.
#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr uint64_t kSelftestWaitNs = 2000000000ull;

__global__ void wait_limit_selftest_kernel(int32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = ptx::smem_addr(&bar);
  ptx::mbar_init(b, 1);
  ptx::fence_mbar_init();
  const uint64_t t0 = ptx::global_timer_ns();
  while (!ptx::mbar_try_wait(b, 0)) {
    if (ptx::global_timer_ns() - t0 > kSelftestWaitNs) {
      atomicCAS(err, 0, kErrWaitTimeout);
      return;
    }
  }
}

}  // namespace

cudaError_t launch_wait_limit_selftest(int32_t* err, cudaStream_t st) {
  wait_limit_selftest_kernel<<<1, 32, 0, st>>>(err);
  return cudaGetLastError();
}

}  // namespace moe
