// Failure-detection self-test for the bounded device waits.
//
// Every wait of the library's tcgen05 kernels on an mbarrier gives up after
// a wall-clock limit, sets an error code and unwinds, so a lost arrival
// (a bug, or a peer that never signals) ends in a status the host can read
// instead of a hung GPU.  This kernel exercises exactly that path: one CTA
// waits on a barrier that nothing will ever signal, with the limit
// shortened by the caller, gives up, writes JSV_ERR_TIMEOUT and exits.
#include "jsv_internal.cuh"
#include "sm100.cuh"

namespace jsv {

__global__ void wait_timeout_selftest_kernel(int32_t *status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_sh;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        abort_sh = 0;
        sm100::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // phase 0 of a fresh barrier with one expected arrival and none coming
        if (!sm100::mbar_wait(&bar, 0, &abort_sh, limit_ns)) atomicCAS(status, 0, JSV_ERR_TIMEOUT);
    }
}

}  // namespace jsv

extern "C" jsv_status jsv_selftest_wait_timeout(int32_t *dev_status, uint32_t limit_us, void *stream) {
    if (!dev_status || limit_us < 1 || limit_us > 2000000) return JSV_ERR_INVALID_ARG;
    jsv::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        dev_status, (uint64_t)limit_us * 1000ull);
    jsv::count_launches(1);
    return cudaGetLastError() == cudaSuccess ? JSV_OK : JSV_ERR_CUDA;
}
