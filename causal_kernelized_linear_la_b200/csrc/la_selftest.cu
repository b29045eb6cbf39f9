// Failure-path self-test of the bounded device-side waits.
//
// Every wait of the tensor-core kernels on an mbarrier is bounded: after its
// limit it records which wait gave up in a device error word and the kernel
// leaves without hanging the GPU; la_prefill_check reports LA_ERR_TIMEOUT.
// A wait can only run out when something upstream failed, so this unit gives
// the failure path a deliberate trigger: one thread waits on an mbarrier that
// nothing arrives at.  No copy or MMA is issued, nothing faults, and the
// context stays usable.
#include "la_internal.cuh"
#include "sm100.cuh"

namespace la {

using namespace sm100;

namespace {

__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel()
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        (void)mbar_wait(&bar, 0, kErrMma);   // gives up after its bound
    }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(cudaStream_t stream)
{
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>();
    return cudaGetLastError();
}

// This unit's copy of the device error word (read and cleared by la_prefill_check).
unsigned int read_and_clear_device_error_selftest(cudaStream_t stream)
{
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return 0;
    cudaStreamSynchronize(stream);
    if (v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
        cudaStreamSynchronize(stream);
    }
    return v;
}

}  // namespace la
