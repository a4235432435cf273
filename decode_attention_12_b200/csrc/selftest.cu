// selftest.cu -- failure-detection self-test of the bounded device waits.
//
// Every wait of the decode and encode kernels (on an mbarrier phase) gives up after
// kWaitLimitNs, records LLA_ERR_DEVICE_TIMEOUT in a status word and lets the kernel wind
// down instead of hanging or trapping.  This kernel exercises exactly that path: its one
// wait is on a barrier that nothing completes, so the wait runs out, the status is
// recorded, the barrier is invalidated and the kernel returns normally.
#include "common.cuh"

namespace lla {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(int32_t *status)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1); // one arrival expected; none will come
        fence_barrier_init();
        if (!mbar_wait_bounded(b, 0))
            report_status(status, LLA_ERR_DEVICE_TIMEOUT);
        asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(b) : "memory");
    }
}

} // namespace
} // namespace lla

extern "C" int lla_selftest_wait_timeout(void *workspace, lla_stream_t stream)
{
    if (workspace == nullptr)
        return LLA_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0)
        return LLA_ERR_MISALIGNED;
    lla::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<int32_t *>(workspace));
    return cudaGetLastError() == cudaSuccess ? LLA_OK : LLA_ERR_CUDA;
}
