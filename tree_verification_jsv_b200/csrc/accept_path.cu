// Greedy accept walk: one warp per request (the walk itself is in walk.cuh).
#include "walk.cuh"

namespace jsv {

constexpr int kWalkWarps = 4;

__global__ void __launch_bounds__(kWalkWarps * 32)
accept_path_kernel(BatchArgs a, const int32_t *__restrict__ tokens,
                   const int32_t *__restrict__ argmax, int max_path, int32_t *__restrict__ path,
                   int32_t *__restrict__ accept_len, int32_t *__restrict__ bonus) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    // the request's parent / token / target-choice arrays, staged once
    __shared__ int32_t s_par[kWalkWarps][kWalkMaxNodes];
    __shared__ int32_t s_tok[kWalkWarps][kWalkMaxNodes];
    __shared__ int32_t s_arg[kWalkWarps][kWalkMaxNodes];
    __shared__ int32_t s_next[kWalkWarps][kWalkMaxNodes];
    const int w = threadIdx.x >> 5;
    const int b = blockIdx.x * kWalkWarps + w;
    const int lane = threadIdx.x & 31;
    if (b >= a.B) return;
    int32_t *row = path + (size_t)b * max_path;

    Request r;
    bool ok = load_request(a, b, r) && r.n <= kWalkMaxNodes;
    if (ok) {
        bool bad = false;
        for (int j = lane; j < r.n; j += 32) {
            const int p = a.parent[r.base + j];
            s_par[w][j] = p;
            s_tok[w][j] = tokens[r.base + j];
            s_arg[w][j] = argmax[r.base + j];
            bad |= (j == 0) ? (p != -1) : (p < 0 || p >= j);
        }
        if (__any_sync(0xffffffffu, bad)) {
            if (lane == 0) flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
            ok = false;
        }
    }
    if (!ok) {
        for (int k = lane; k < max_path; k += 32) row[k] = k == 0 ? 0 : -1;
        if (lane == 0) { accept_len[b] = 0; bonus[b] = -1; }
        return;
    }
    __syncwarp();

    int last = 0;
    bool cut = false;
    const int len = greedy_walk_warp(s_par[w], s_tok[w], s_arg[w], s_next[w], r.n, max_path, row, lane, last, cut);
    if (cut && lane == 0) flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
    if (lane == 0) {
        row[0] = 0;
        accept_len[b] = len - 1;
        bonus[b] = s_arg[w][last];
    }
    for (int k = len + lane; k < max_path; k += 32) row[k] = -1;
}

cudaError_t launch_accept_path(const BatchArgs &a, const int32_t *tokens, const int32_t *argmax,
                               int max_path, int32_t *path, int32_t *accept_len, int32_t *bonus,
                               cudaStream_t st) {
    dim3 grid((a.B + kWalkWarps - 1) / kWalkWarps);
    static PerDeviceOnce carve;
    cudaError_t e = prefer_max_shared(accept_path_kernel, carve);
    if (e != cudaSuccess) return e;
    e = launch_pdl(accept_path_kernel, grid, dim3(kWalkWarps * 32), 0, st, a, tokens, argmax, max_path,
                               path, accept_len, bonus);
    count_launches(1);
    return e;
}

}  // namespace jsv
