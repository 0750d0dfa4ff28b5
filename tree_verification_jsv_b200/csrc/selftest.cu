// Failure-detection self-tests for the bounded device waits.
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

// The LM head with one injected wait that gives up (see jsv.h): the same
// launch as jsv_lmhead_argmax (workspace given) or jsv_lmhead_argmax_noalloc
// (workspace NULL), with the first CTA's producer stalled on a barrier that
// nothing signals before it issues any copy.
extern "C" jsv_status jsv_selftest_lmhead_timeout(const uint16_t *hidden, const uint16_t *w, int32_t T, int32_t d,
                                                  int32_t V, int32_t *argmax, float *max_logit, void *workspace,
                                                  size_t workspace_bytes, int32_t *dev_status, uint32_t limit_us,
                                                  void *stream) {
    jsv_status s = jsv::check_lmhead_args(hidden, w, T, d, V, argmax);
    if (s != JSV_OK) return s;
    if (!dev_status || limit_us < 1 || limit_us > 2000000) return JSV_ERR_INVALID_ARG;
    if (workspace) {
        if (workspace_bytes < jsv::lmhead_workspace_bytes(T, d, V) ||
            (reinterpret_cast<uintptr_t>(workspace) % 8) != 0)
            return JSV_ERR_INVALID_ARG;
    } else {
        if (T > JSV_NOALLOC_MAX_NODES) return JSV_ERR_UNSUPPORTED;
        s = jsv::from_cuda(jsv::noalloc_scratch(&workspace));
        if (s != JSV_OK) return s;
    }
    return jsv::from_cuda(jsv::launch_lmhead_argmax(hidden, w, T, d, V, argmax, max_logit, workspace, dev_status,
                                                    (uint64_t)limit_us * 1000ull, static_cast<cudaStream_t>(stream)));
}
