// diag.cu -- diagnostics of the library's failure handling that need no fault: a wait that runs out.
#include "launch.cuh"

namespace msa {

// One thread waits on a shared-memory barrier that nothing arrives on, bounded like every wait of
// the library's kernels (here by limit_ns); when the bound runs out it reports MSA_DERR_TIMEOUT.
__global__ void wait_timeout_probe_kernel(int *err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        if (!mbar_wait_limit(&bar, 0, limit_ns)) report(err, kErrTimeout);
    }
}

cudaError_t launch_wait_timeout_probe(int *err, uint64_t limit_ns, cudaStream_t st) {
    wait_timeout_probe_kernel<<<1, 32, 0, st>>>(err, limit_ns);
    return cudaGetLastError();
}

}  // namespace msa
