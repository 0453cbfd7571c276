// Self-test of the failure path every pipelined kernel shares: a bounded mbarrier wait that runs
// out raises the device error word and returns, leaving the context usable.
#include "sm100.cuh"

namespace qg {
namespace {

// One thread waits on a barrier that nothing ever arrives on; the wait gives up after
// limit_ns, sets the error word (read and cleared by qgemm_sync_check) and the kernel returns.
__global__ void wait_selftest_kernel(unsigned int *err, unsigned long long limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, err, limit_ns);
}

} // namespace

cudaError_t launch_wait_selftest(unsigned int *err, unsigned long long limit_ns,
                                 cudaStream_t stream)
{
    wait_selftest_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
    return cudaGetLastError();
}

} // namespace qg
