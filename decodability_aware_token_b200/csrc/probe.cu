// Failure-path probe: shows that a pipeline wait that is never satisfied ends with an error status
// instead of hanging the GPU.  One CTA initialises an mbarrier that nothing will complete and waits on
// it with the same bounded wait the GEMM and attention pipelines use; after about a second the wait
// gives up, sets FOCUS_DEVERR_TIMEOUT in the context's error word and the kernel returns.  No trap, no
// fault: the context stays usable.
#include "launch.h"
#include "tc_gemm_kernel.cuh"

namespace focus {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_probe_kernel(int* err) {
    __shared__ __align__(8) uint64_t never;
    if (threadIdx.x == 0) {
        tc::mbar_init(&never, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if (threadIdx.x == 0) tc::mbar_wait(&never, 0u, err);  // nobody arrives: the bounded wait expires
}

}  // namespace

int launch_wait_timeout_probe(int* err, cudaStream_t s) {
    wait_timeout_probe_kernel<<<1, 32, 0, s>>>(err);
    return cudaGetLastError() == cudaSuccess ? 1 : -1;
}

}  // namespace focus
