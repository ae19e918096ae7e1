// selftest.cu -- exercises the bounded mbarrier wait that every kernel wait
// uses: one CTA waits on a barrier that nobody arrives at and must give up
// after the limit, set the timeout flag in the status word and return.  It
// neither hangs nor faults the GPU.
#include <cstdint>

#include "sm100.cuh"

namespace smla {

__global__ void selftest_wait_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait_bounded(&bar, 0, limit_ns, status);
}

}  // namespace smla
