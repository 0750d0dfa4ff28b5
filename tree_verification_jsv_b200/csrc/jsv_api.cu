// C ABI of libjsv.so: host-side argument checks, then one launch sequence
// per call on the caller's stream.  See include/jsv.h for the contract.
#include "jsv_internal.cuh"

#include <atomic>
#include <cstdio>

namespace jsv {
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static thread_local char t_launch_note[256] = {0};
void note_launch_failure(const char *what, int regs, int max_threads, size_t static_smem, int max_dyn_smem,
                         int threads, size_t dyn_smem) {
    snprintf(t_launch_note, sizeof t_launch_note,
             "%s launch: %d regs/thread, max %d threads/block, %zu B static + %zu B dynamic smem "
             "requested (limit %d B dynamic), %d threads",
             what, regs, max_threads, static_smem, dyn_smem, max_dyn_smem, threads);
}
}  // namespace jsv

namespace {

bool aligned(const void *p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

jsv_status check_batch(const jsv_batch *b) {
    if (!b) return JSV_ERR_INVALID_ARG;
    if (b->B < 1 || b->Hq < 1 || b->Hkv < 1 || b->total_nodes < b->B || b->max_nodes < 1 ||
        b->max_prefix < 0 || b->max_pages_per_req < 1 || b->num_pages < 1)
        return JSV_ERR_INVALID_ARG;
    if (b->Hq % b->Hkv != 0) return JSV_ERR_INVALID_ARG;
    if (b->D != 64 && b->D != 128) return JSV_ERR_UNSUPPORTED;
    if (b->page_size != 16) return JSV_ERR_UNSUPPORTED;
    if (b->max_nodes > 512) return JSV_ERR_UNSUPPORTED;
    if ((long long)b->max_pages_per_req * b->page_size < 1) return JSV_ERR_INVALID_ARG;
    if (!b->page_table || !b->prefix_len || !b->node_offsets || !b->parent) return JSV_ERR_INVALID_ARG;
    return JSV_OK;
}

}  // namespace

namespace jsv {
thread_local cudaError_t t_last_error = cudaSuccess;

jsv_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return JSV_OK;
    t_last_error = e;
    return JSV_ERR_CUDA;
}

jsv_status check_lmhead_args(const uint16_t *hidden, const uint16_t *w, int32_t T, int32_t d, int32_t V,
                             const int32_t *argmax) {
    if (!hidden || !w || !argmax || T < 1 || d < 1 || V < 1) return JSV_ERR_INVALID_ARG;
    if (d % 64 != 0 || d > 16384) return JSV_ERR_UNSUPPORTED;
    if (!aligned(hidden, 16) || !aligned(w, 16)) return JSV_ERR_INVALID_ARG;
    return JSV_OK;
}
}  // namespace jsv

using jsv::from_cuda;

extern "C" {

size_t jsv_tree_attention_workspace_size(const jsv_batch *batch) {
    if (check_batch(batch) != JSV_OK) return 0;
    return jsv::attention_workspace_bytes(jsv::to_args(batch));
}

jsv_status jsv_tree_attention(const jsv_batch *batch, const uint16_t *q, const uint16_t *k_cache,
                              const uint16_t *v_cache, float scale, uint16_t *out, void *workspace,
                              size_t workspace_bytes, void *stream) {
    jsv_status s = check_batch(batch);
    if (s != JSV_OK) return s;
    if (!q || !k_cache || !v_cache || !out) return JSV_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16))
        return JSV_ERR_INVALID_ARG;
    if (!(scale > 0.f) || scale != scale) return JSV_ERR_INVALID_ARG;
    const jsv::BatchArgs a = jsv::to_args(batch);
    const size_t need = jsv::attention_workspace_bytes(a);
    if (workspace_bytes < need || (need && (!workspace || !aligned(workspace, 256))))
        return JSV_ERR_INVALID_ARG;
    return from_cuda(jsv::launch_tree_attention(a, q, k_cache, v_cache, scale, out, workspace,
                                                static_cast<cudaStream_t>(stream)));
}

size_t jsv_lmhead_argmax_workspace_size(int32_t T, int32_t d, int32_t V) {
    if (T < 1 || d < 1 || V < 1) return 0;
    return jsv::lmhead_workspace_bytes(T, d, V);
}

jsv_status jsv_lmhead_argmax(const uint16_t *hidden, const uint16_t *w, int32_t T, int32_t d,
                             int32_t V, int32_t *argmax, float *max_logit, void *workspace,
                             size_t workspace_bytes, int32_t *dev_status, void *stream) {
    jsv_status s = jsv::check_lmhead_args(hidden, w, T, d, V, argmax);
    if (s != JSV_OK) return s;
    const size_t need = jsv::lmhead_workspace_bytes(T, d, V);
    if (workspace_bytes < need || !workspace || !aligned(workspace, 8)) return JSV_ERR_INVALID_ARG;
    return from_cuda(jsv::launch_lmhead_argmax(hidden, w, T, d, V, argmax, max_logit, workspace, dev_status, 0,
                                               static_cast<cudaStream_t>(stream)));
}

jsv_status jsv_accept_path(const jsv_batch *batch, const int32_t *tokens, const int32_t *argmax,
                           int32_t max_path, int32_t *path, int32_t *accept_len, int32_t *bonus,
                           void *stream) {
    jsv_status s = check_batch(batch);
    if (s != JSV_OK) return s;
    if (!tokens || !argmax || !path || !accept_len || !bonus || max_path < 1) return JSV_ERR_INVALID_ARG;
    return from_cuda(jsv::launch_accept_path(jsv::to_args(batch), tokens, argmax, max_path, path,
                                             accept_len, bonus, static_cast<cudaStream_t>(stream)));
}

jsv_status jsv_kv_compact(const jsv_batch *batch, uint16_t *k_cache, uint16_t *v_cache,
                          const int32_t *path, int32_t max_path, const int32_t *accept_len,
                          int32_t *new_len, void *stream) {
    jsv_status s = check_batch(batch);
    if (s != JSV_OK) return s;
    if (!k_cache || !v_cache || !path || !accept_len || !new_len || max_path < 1)
        return JSV_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return JSV_ERR_INVALID_ARG;
    return from_cuda(jsv::launch_kv_compact(jsv::to_args(batch), k_cache, v_cache, path, max_path,
                                            accept_len, new_len, static_cast<cudaStream_t>(stream)));
}

jsv_status jsv_accept_compact(const jsv_batch *batch, const int32_t *tokens, const int32_t *argmax,
                              int32_t max_path, int32_t *path, int32_t *accept_len, int32_t *bonus,
                              uint16_t *k_cache, uint16_t *v_cache, int32_t *new_len, void *stream) {
    jsv_status s = check_batch(batch);
    if (s != JSV_OK) return s;
    if (!tokens || !argmax || !path || !accept_len || !bonus || !k_cache || !v_cache || !new_len || max_path < 1)
        return JSV_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return JSV_ERR_INVALID_ARG;
    return from_cuda(jsv::launch_accept_compact(jsv::to_args(batch), tokens, argmax, max_path, path, accept_len,
                                                bonus, k_cache, v_cache, new_len, static_cast<cudaStream_t>(stream)));
}

jsv_status jsv_tree_qkv_rope(const jsv_batch *batch, const uint16_t *x, const uint16_t *w_qkv, int32_t d,
                             const float *rope_cos, const float *rope_sin, int32_t max_pos, uint16_t *q,
                             uint16_t *k_cache, uint16_t *v_cache, void *stream) {
    jsv_status s = check_batch(batch);
    if (s != JSV_OK) return s;
    if (!x || !w_qkv || !rope_cos || !rope_sin || !q || !k_cache || !v_cache || max_pos < 1 || d < 1)
        return JSV_ERR_INVALID_ARG;
    if (d % 64 != 0 || d > 16384) return JSV_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return JSV_ERR_INVALID_ARG;
    return from_cuda(jsv::launch_tree_qkv_rope(jsv::to_args(batch), x, w_qkv, d, rope_cos, rope_sin, max_pos, q,
                                               k_cache, v_cache, static_cast<cudaStream_t>(stream)));
}

jsv_status jsv_accum_logp_tree(const float *logp, const int32_t *topk_tokens, const int32_t *root_token,
                               int32_t B, int32_t depth, int32_t width, int32_t budget, int32_t *parent,
                               int32_t *tokens, int32_t *node_depth, float *score, int32_t *num_nodes,
                               int32_t *dev_status, void *stream) {
    if (B < 1 || depth < 0 || width < 1 || budget < 1) return JSV_ERR_INVALID_ARG;
    if (depth > 32 || width > 32 || budget > 512) return JSV_ERR_UNSUPPORTED;
    if ((depth > 0 && (!logp || !topk_tokens)) || !root_token || !parent || !tokens || !node_depth || !num_nodes)
        return JSV_ERR_INVALID_ARG;
    return from_cuda(jsv::launch_accum_logp_tree(logp, topk_tokens, root_token, B, depth, width, budget, parent,
                                                 tokens, node_depth, score, num_nodes, dev_status,
                                                 static_cast<cudaStream_t>(stream)));
}

const char *jsv_status_string(jsv_status status) {
    switch (status) {
        case JSV_OK: return "ok";
        case JSV_ERR_INVALID_ARG: return "invalid argument";
        case JSV_ERR_UNSUPPORTED: return "unsupported shape";
        case JSV_ERR_CUDA: return "CUDA error";
        case JSV_ERR_TIMEOUT: return "device wait timed out";
        case JSV_ERR_DEVICE_INPUT: return "malformed device-side input";
        case JSV_ERR_BOUNDS: return "index out of bounds (checked build)";
    }
    return "unknown status";
}

int32_t jsv_version(void) { return 100; }

int32_t jsv_build_flags(void) {
#ifdef JSV_CHECK_BOUNDS
    return 1;
#else
    return 0;
#endif
}

const char *jsv_last_error_string(void) {
    static thread_local char buf[512];
    if (jsv::t_last_error == cudaSuccess) return "no CUDA error recorded";
    snprintf(buf, sizeof buf, "%s%s%s", cudaGetErrorString(jsv::t_last_error), jsv::t_launch_note[0] ? " -- " : "",
             jsv::t_launch_note);
    return buf;
}

uint64_t jsv_kernel_launches(void) { return jsv::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
