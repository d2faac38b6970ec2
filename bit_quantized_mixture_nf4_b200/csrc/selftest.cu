// Watchdog self-test: one thread waits on an mbarrier that nothing will ever
// arrive at, through the same bounded wait every pipelined kernel uses.  After
// the wait's time limit (2 s) it records the timeout in the device status word
// and returns; nothing faults, traps or hangs, and the context stays usable.
#include "../../include/e4b.h"
#include "e4b_internal.h"

namespace e4b {

__global__ void watchdog_selftest_kernel(uint32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_u32(&bar);
    abort_flag = 0;
    mbar_init(b, 1);   // one arrival expected, none will come
    fence_barrier_init();
    mbar_wait(b, 0, &abort_flag, status);
}

}  // namespace e4b

extern "C" e4b_status e4b_watchdog_selftest(void* stream) {
    uint32_t* status = e4b::device_status_ptr();
    if (!status) return E4B_ERR_CUDA;
    e4b::watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status);
    e4b::count_launch();
    return cudaGetLastError() == cudaSuccess ? E4B_OK : E4B_ERR_CUDA;
}
