// LM-head argmax without caller-provided or library-allocated scratch.
//
// Some callers cannot allocate device memory at the point where they run
// the verify step: code that runs inside a CUDA-graph-captured region or an
// allocator-less embedding (a plugin loaded by an inference server that
// owns every allocation, a custom memory pool that forbids foreign
// cudaMalloc, a latency-critical loop where cudaMalloc's implicit
// synchronisation is unacceptable).  For them this file provides one extra
// entry point whose scratch -- one 64-bit argmax key per node -- lives in a
// fixed file-scope device array instead of a workspace argument.
//
// The array is JSV_NOALLOC_MAX_NODES keys plus one counter word (64 KiB + 8 B).  Every GPU that loads
// the library holds it until the process exits.  Host code must not pass
// the array's name to a kernel (on the host it is only a stand-in for the
// symbol); its device address is looked up once per device, with that
// device current, by cudaGetSymbolAddress, and cached.
#include "jsv_internal.cuh"

#include <mutex>

namespace jsv {

// one 64-bit argmax key per node plus the LM-head kernel's completion counter
static __device__ __align__(256) unsigned long long g_lmhead_noalloc_keys[JSV_NOALLOC_MAX_NODES + 1];

namespace {
std::mutex g_noalloc_mu;
void *g_noalloc_addr[64] = {nullptr};
}  // namespace

// Device address of the scratch array on the current device (set-up on the
// first call made with that device current).
cudaError_t noalloc_scratch(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_lmhead_noalloc_keys);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}

}  // namespace jsv

extern "C" {

jsv_status jsv_lmhead_argmax_noalloc(const uint16_t *hidden, const uint16_t *w, int32_t T, int32_t d,
                                     int32_t V, int32_t *argmax, float *max_logit, int32_t *dev_status,
                                     void *stream) {
    jsv_status s = jsv::check_lmhead_args(hidden, w, T, d, V, argmax);
    if (s != JSV_OK) return s;
    if (T > JSV_NOALLOC_MAX_NODES) return JSV_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    s = jsv::from_cuda(jsv::noalloc_scratch(&scratch));
    if (s != JSV_OK) return s;
    // the array is zero at load and every call leaves its keys and counter
    // zeroed, a call that timed out included
    static_assert(sizeof(jsv::g_lmhead_noalloc_keys) >= (JSV_NOALLOC_MAX_NODES + 1) * sizeof(unsigned long long),
                  "scratch must hold the keys and the completion counter");
    return jsv::from_cuda(jsv::launch_lmhead_argmax(hidden, w, T, d, V, argmax, max_logit, scratch, dev_status, 0,
                                                    static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
