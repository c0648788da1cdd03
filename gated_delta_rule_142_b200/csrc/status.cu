// status.cu -- device-side failure reporting.
//
// Every wait inside the library's kernels is a bounded mbarrier.try_wait loop.
// When one gives up, the kernel raises an abort flag that releases its other
// waits, frees its tensor memory, sets a device error word and returns; its
// results are then wrong but nothing hangs.  gdn_device_status() (gdn_api.cu)
// reads and clears those words.  The self-test below exercises the same path
// on purpose: one thread waits, with a short bound, on an mbarrier phase that
// no one completes, gives up and sets its word.
#include "gdn.h"
#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

__device__ int g_selftest_timeout;

__global__ void selftest_timeout_kernel(unsigned iters) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bool done = false;
        for (unsigned i = 0; i < iters && !done; ++i) done = sm100::mbar_try_wait(&bar, 0);
        if (!done) atomicExch(&g_selftest_timeout, 1);
    }
}

}  // namespace

cudaError_t launch_selftest_timeout(cudaStream_t stream) {
    selftest_timeout_kernel<<<1, 32, 0, stream>>>(1u << 12);
    return cudaGetLastError();
}

bool take_selftest_timeout() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_selftest_timeout, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_selftest_timeout, &zero, sizeof(int));
    }
    return v != 0;
}

}  // namespace gdn
