// Failure-path self-test of the library's bounded device-side waits.
//
// Every tensor-core kernel hands work between warps through mbarriers whose
// waits give up after a time limit, record MM_ERR_TIMEOUT in the device status
// word and let the CTA finish, so that a stalled pipeline surfaces as an error
// code instead of a hung GPU.  mm_selftest_wait_timeout runs that path on
// purpose: one CTA waits on an mbarrier that nothing arrives on, through the
// same wait helper and with a caller-given limit, then returns.
#include "mm_internal.cuh"
#include "sm100.cuh"

namespace mm {
namespace {

using namespace sm100;

__global__ void selftest_wait_kernel(uint64_t limit_ns, int* status)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // one arrival expected; none comes
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar, 0, &abort_flag, limit_ns));
    if (!ok && threadIdx.x == 0) raise_timeout(&abort_flag, status);
}

}  // namespace
}  // namespace mm

extern "C" int mm_selftest_wait_timeout(unsigned timeout_us, void* stream)
{
    if (timeout_us == 0 || timeout_us > 1000000u) return MM_ERR_SHAPE;
    mm::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)timeout_us * 1000u,
                                                                                mm::device_status_ptr());
    return cudaGetLastError() == cudaSuccess ? MM_OK : MM_ERR_CUDA;
}
