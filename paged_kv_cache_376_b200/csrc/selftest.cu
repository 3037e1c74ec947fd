// Self-test of the bounded waits every kernel of the library relies on.
//
// Every spin in libtv is an mbarrier wait that gives up after a limit of
// %globaltimer time, sets TV_DEVERR_TIMEOUT in the caller's error word and
// lets the kernel return, so a lost copy or a missing arrive can never hang
// the GPU.  This kernel exercises that path for real: one thread waits on an
// mbarrier that nothing will ever complete, with a short limit, and must
// come back with the time-out flagged.  No fault, trap or endless loop is
// involved; the context stays usable.
#include "tv_device.cuh"
#include "tv_kernels.h"

namespace tv {
namespace {

__global__ void wait_selftest_kernel(uint32_t* err,
                                     unsigned long long limit_ns,
                                     unsigned long long* waited_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_mbar_init();
  // wait for phase 0, which nothing completes
  const unsigned long long t0 = global_timer_ns();
  bool done = mbar_try_wait(b, 0);
  while (!done && global_timer_ns() - t0 <= limit_ns) done = mbar_try_wait(b, 0);
  const unsigned long long t1 = global_timer_ns();
  if (!done) flag_error(err, DEVERR_TIMEOUT);
  if (waited_ns) *waited_ns = t1 - t0;
}

}  // namespace

cudaError_t launch_wait_selftest(uint32_t* err, unsigned long long limit_ns,
                                 unsigned long long* waited_ns,
                                 cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns, waited_ns);
  return cudaGetLastError();
}

}  // namespace tv
