// Internal helpers shared by the libjsv.so kernels (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/jsv.h"

namespace jsv {

// Device-side copy of the host-visible batch geometry (passed by value).
struct BatchArgs {
    int B, Hq, Hkv, D, page_size, max_pages_per_req, num_pages, total_nodes, max_nodes, max_prefix;
    const int32_t *page_table, *prefix_len, *node_offsets, *parent;
    int32_t *dev_status;
};

inline BatchArgs to_args(const jsv_batch *b) {
    BatchArgs a;
    a.B = b->B; a.Hq = b->Hq; a.Hkv = b->Hkv; a.D = b->D; a.page_size = b->page_size;
    a.max_pages_per_req = b->max_pages_per_req; a.num_pages = b->num_pages;
    a.total_nodes = b->total_nodes; a.max_nodes = b->max_nodes; a.max_prefix = b->max_prefix;
    a.page_table = b->page_table; a.prefix_len = b->prefix_len; a.node_offsets = b->node_offsets;
    a.parent = b->parent; a.dev_status = b->dev_status;
    return a;
}

// One-time host set-up per device (kernel attributes): the first call made
// with a device current runs it under a lock, later calls read a flag, so
// host threads that make their first calls at the same time do not race.  A
// set-up that failed is not recorded and runs again on the next call.
// Devices past the table run it on every call.
class PerDeviceOnce {
public:
    template <typename F>
    cudaError_t run(F &&f) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kDevices) return f();
        if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lock(mu_);
        if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        e = f();
        if (e == cudaSuccess) done_[dev].store(true, std::memory_order_release);
        return e;
    }

private:
    static constexpr int kDevices = 64;
    std::atomic<bool> done_[kDevices] = {};
    std::mutex mu_;
};

// Kernels of a step run side by side on one SM (programmatic dependent
// launch lets the next kernel start early), but an SM's split between L1 and
// shared memory stays fixed while any CTA is resident on it.  A small kernel
// left to the driver's default split would take a large L1 and keep the
// LM-head and attention CTAs, which need most of the shared memory, off every
// SM it occupies until it exits.  So every kernel asks for the largest shared
// carveout, once per device.
template <typename K>
inline cudaError_t prefer_max_shared(K *kernel, PerDeviceOnce &once) {
    return once.run([&]() {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                    (int)cudaSharedmemCarveoutMaxShared);
    });
}

// Programmatic dependent launch: every kernel of the library is launched so
// that the next kernel in the stream may be scheduled before it finishes.
// A kernel lets its dependents be scheduled at entry (they can only start
// once every CTA of this grid has started or exited, so they never take SMs
// this grid still needs), and waits for its own predecessor to complete --
// and its memory to be visible -- before it reads any input.
__device__ __forceinline__ void pdl_allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_predecessor() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void flag_error(int32_t *status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Index checks of the checked build (-DJSV_CHECK_BOUNDS, libjsv_checked.so):
// a computed global index is compared with its buffer's extent before the
// access, and one outside records JSV_ERR_BOUNDS in the status word and the
// access is skipped.  The kernels' own input checks keep every index in
// range, so a failure here is a fault of the library.  In the ordinary
// build the check is `true` and costs nothing.
#ifdef JSV_CHECK_BOUNDS
__device__ __forceinline__ bool index_ok(long long i, long long n, int32_t *status) {
    if (i >= 0 && i < n) return true;
    flag_error(status, JSV_ERR_BOUNDS);
    return false;
}
#define JSV_IN_BOUNDS(i, n, status) ::jsv::index_ok((long long)(i), (long long)(n), (status))
#else
#define JSV_IN_BOUNDS(i, n, status) ((void)(i), (void)(n), true)
#endif

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h) {
    return __uint_as_float(((uint32_t)h) << 16);
}

// Request geometry read from device arrays, with the checks every kernel
// needs before touching the request's memory.  Returns false (and flags the
// status word) if the request's descriptors are inconsistent.
struct Request {
    int base, n, P;
};

__device__ __forceinline__ bool load_request(const BatchArgs &a, int b, Request &r) {
    if (!JSV_IN_BOUNDS(b, a.B, a.dev_status)) return false;
    int s = a.node_offsets[b], e = a.node_offsets[b + 1];
    int P = a.prefix_len[b];
    bool ok = s >= 0 && e > s && e <= a.total_nodes && (e - s) <= a.max_nodes &&
              P >= 0 && P <= a.max_prefix &&
              (P + (e - s) + a.page_size - 1) / a.page_size <= a.max_pages_per_req;
    if (b == a.B - 1 && e != a.total_nodes) ok = false;
    if (!ok) {
        flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
        return false;
    }
    r.base = s; r.n = e - s; r.P = P;
    return true;
}

// Physical row index (page * page_size + offset) of logical slot s, or -1
// (flagged) if the page entry is out of range.
__device__ __forceinline__ long long slot_phys_row(const BatchArgs &a, int b, int s) {
    const long long pi = (long long)b * a.max_pages_per_req + s / a.page_size;
    if (!JSV_IN_BOUNDS(pi, (long long)a.B * a.max_pages_per_req, a.dev_status)) return -1;
    int page = a.page_table[pi];
    if (page < 0 || page >= a.num_pages) {
        flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
        return -1;
    }
    return (long long)page * a.page_size + (s % a.page_size);
}

// Count of kernel launches issued by the library (see jsv_kernel_launches).
void count_launches(int n);

// Host-side status of a CUDA call (records the error for jsv_last_error_string).
jsv_status from_cuda(cudaError_t e);

// Host-side checks shared by the LM-head entry points.
jsv_status check_lmhead_args(const uint16_t *hidden, const uint16_t *w, int32_t T, int32_t d, int32_t V,
                             const int32_t *argmax);

// Device address of the allocation-free LM head's scratch array on the
// current device (looked up with that device current on first use).
cudaError_t noalloc_scratch(void **out);

// Record the resources of a kernel whose launch failed, for
// jsv_last_error_string (thread-local).
void note_launch_failure(const char *what, int regs, int max_threads, size_t static_smem, int max_dyn_smem,
                         int threads, size_t dyn_smem);

// Launch `kernel` on `st` with programmatic stream serialization allowed.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Same, with thread-block clusters of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      int cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace jsv

// Launchers (defined in the kernel files, called from jsv_api.cu).
namespace jsv {
cudaError_t launch_accept_path(const BatchArgs &a, const int32_t *tokens, const int32_t *argmax,
                               int max_path, int32_t *path, int32_t *accept_len, int32_t *bonus,
                               cudaStream_t st);
cudaError_t launch_kv_compact(const BatchArgs &a, uint16_t *k_cache, uint16_t *v_cache,
                              const int32_t *path, int max_path, const int32_t *accept_len,
                              int32_t *new_len, cudaStream_t st);
cudaError_t launch_accept_compact(const BatchArgs &a, const int32_t *tokens, const int32_t *argmax, int max_path,
                                  int32_t *path, int32_t *accept_len, int32_t *bonus, uint16_t *k_cache,
                                  uint16_t *v_cache, int32_t *new_len, cudaStream_t st);
size_t lmhead_workspace_bytes(int T, int d, int V);
// status: device status word or NULL; inject_ns: 0, or the limit of the
// failure-detection self-test's injected wait (jsv_selftest_lmhead_timeout)
cudaError_t launch_lmhead_argmax(const uint16_t *hidden, const uint16_t *w, int T, int d, int V,
                                 int32_t *argmax, float *max_logit, void *ws, int32_t *status,
                                 uint64_t inject_ns, cudaStream_t st);
size_t attention_workspace_bytes(const BatchArgs &a);
cudaError_t launch_tree_qkv_rope(const BatchArgs &a, const uint16_t *x, const uint16_t *w_qkv, int d,
                                 const float *rope_cos, const float *rope_sin, int max_pos, uint16_t *q,
                                 uint16_t *k_cache, uint16_t *v_cache, cudaStream_t st);
cudaError_t launch_accum_logp_tree(const float *logp, const int32_t *topk_tokens, const int32_t *root_token, int B,
                                   int D, int k, int budget, int32_t *parent, int32_t *tokens, int32_t *depth,
                                   float *score, int32_t *num_nodes, int32_t *status, cudaStream_t st);
cudaError_t launch_tree_attention(const BatchArgs &a, const uint16_t *q, const uint16_t *k_cache,
                                  const uint16_t *v_cache, float scale, uint16_t *out, void *ws,
                                  cudaStream_t st);
}  // namespace jsv
