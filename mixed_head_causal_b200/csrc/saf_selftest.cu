// Failure-path self-test: a device-side wait that nothing completes.
//
// Every wait in the kernels is bounded; one that gives up records an error
// word in the workspace header, which saf_device_status reports as a time-out
// and clears.  This kernel exercises that path on the GPU without a fault: one
// thread waits on an mbarrier that expects an arrival nobody makes, gives up
// after `limit` cycles (no copies or MMAs are in flight), reports, and returns.
#include "saf_common.cuh"
#include "tc_util.cuh"

namespace saf {
namespace {

__global__ void selftest_wait_kernel(unsigned int* err, long long limit) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = tc::smem_addr(&bar);
    if (threadIdx.x == 0) {
        tc::mbar_init(b, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !tc::mbar_wait(b, 0, limit)) {
        atomicOr(err, 1u);
        atomicCAS(err + 1, 0u, 0xF001u);
    }
}

}  // namespace

cudaError_t launch_selftest_wait(unsigned int* err, long long limit, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>(err, limit);
    return cudaGetLastError();
}

}  // namespace saf
