// selftest.cu -- exercises the bounded-wait failure path on the device.
//
// Every kernel of this library waits on mbarriers through wait_or_abort(), which gives up after a
// limit of SM clock cycles, records MSA_ERR_TIMEOUT (with the waiting site) in the device error
// word and lets the kernel return instead of hanging. This kernel runs that routine on a barrier
// phase that nothing ever completes, with a caller-chosen short limit, so that a test can check
// the whole path (the wait expires, the status reaches the host, the context stays usable)
// without faulting or hanging the GPU.
#include "common.cuh"
#include "sm100.cuh"

namespace msa {

namespace {

constexpr int kSelftestSite = 900;

__global__ void __launch_bounds__(32, 1) selftest_wait_kernel(int* err, long long limit)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1); // expects one arrival that never comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) wait_or_abort(&bar, 0, &abort_flag, err, kSelftestSite, limit);
}

} // namespace

cudaError_t launch_selftest_wait(int* err, long long limit_cycles, cudaStream_t s)
{
    selftest_wait_kernel<<<1, 32, 0, s>>>(err, limit_cycles);
    note_launch(1);
    return cudaGetLastError();
}

} // namespace msa
