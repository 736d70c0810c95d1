// Self-test of the bounded-wait mechanism every pipeline wait of the library
// uses: one thread waits on an mbarrier that nothing arrives at, gives up
// after `limit_ns` of %globaltimer, ORs BSA_DEV_TIMEOUT into the status word
// and returns, so the context stays usable.  Nothing else runs.
#include "internal.cuh"
#include "sm100.cuh"

namespace bsa {
namespace {

__global__ void wait_selftest_kernel(int32_t* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = sm100::globaltimer_ns();
    while (!sm100::mbar_test(&bar, 0)) {
      if (sm100::globaltimer_ns() - t0 > limit_ns) {
        atomicOr(status, BSA_DEV_TIMEOUT);
        break;
      }
    }
  }
}

}  // namespace

cudaError_t launch_wait_selftest(int32_t* status, unsigned long long limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace bsa
