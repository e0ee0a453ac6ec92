// selftest.cu -- exercise of the bounded-wait failure path on the device.
//
// One CTA initialises an mbarrier that nothing ever arrives on and waits for
// it with the library's bounded wait.  The wait gives up after
// IC_WAIT_LIMIT_NS, sets IC_DEV_TIMEOUT in the status word and the kernel
// returns normally, so the context stays usable.  This is the same wait every
// pipeline of the library uses; the entry point lets a test check, without
// faulting or hanging anything, that a stalled pipeline ends with a status
// the host can read.
#include "sm100.cuh"

namespace ic {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort_flag = 0;
        sm100::fence_mbar_init();
    }
    __syncwarp();
    // phase 0 never completes: no thread arrives on `bar`
    sm100::warp_wait(&bar, 0, status, &abort_flag);
}

}  // namespace
}  // namespace ic

extern "C" ic_status ic_selftest_wait_timeout(void* ws, size_t ws_bytes, void* stream) {
    if (ws == nullptr || ws_bytes < IC_STATUS_BYTES || ((uintptr_t)ws & 255)) return IC_ERR_INVALID_ARG;
    ic::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<uint32_t*>(ws));
    return ic::last_launch_status();
}
