// selftest.cu -- exercises the kernels' bounded waits without any fault: one
// CTA waits on an mbarrier that nothing arrives on and on a global counter
// that nothing raises, each for a short limit, and reports the expiry
// through dev_status exactly as the decode kernel's roles do.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/nvfp4mla.h"
#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4mla {
using namespace ptx;

__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(uint32_t *counter, unsigned long long max_cycles,
                                                             int32_t *dev_status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    const bool bar_done = mbar_wait(&bar, 0, max_cycles);       // nobody arrives
    const bool cnt_done = spin_until_geq(counter, 1u, max_cycles);  // nobody raises it
    if (!bar_done && !cnt_done) atomicOr(dev_status, NVFP4MLA_DEV_TIMEOUT);
    mbar_arrive(&bar);  // complete the phase so the barrier is left consistent
}

cudaError_t launch_wait_timeout_selftest(uint32_t *counter, int32_t *dev_status, cudaStream_t stream) {
    // ~1 ms at the B200's 1.9 GHz clock for each of the two waits
    wait_timeout_kernel<<<1, 32, 0, stream>>>(counter, 2000000ull, dev_status);
    return cudaGetLastError();
}

}  // namespace nvfp4mla
