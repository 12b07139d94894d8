// probe.cu -- a kernel whose only job is to let a bounded device-side wait
// run out: one thread waits on an mbarrier that nothing arrives on, gives up
// after the requested time and records CSA_ERR_TIMEOUT in the device error
// word, exactly as the pipeline kernels do when one of their waits expires.
// It issues no copy and no tensor-core work, so nothing is in flight when it
// returns and the context stays usable.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace csa {

namespace {

__global__ void wait_probe_kernel(uint64_t limit_ns, unsigned *err)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile int never = 0;
        if (!tc::mbar_wait(&bar, 0, &never, limit_ns))
            report(err, CSA_ERR_TIMEOUT, K_PROBE, 0, 0);
    }
}

}  // namespace

cudaError_t launch_wait_probe(uint64_t limit_ns, unsigned *err, cudaStream_t s)
{
    wait_probe_kernel<<<1, 32, 0, s>>>(limit_ns, err);
    return cudaGetLastError();
}

}  // namespace csa
