// Accepted-path KV compaction, in place in the paged cache.
//
// Paged KV per the JetSpec README ("JetSpec / Quick Start"); the ragged
// batch motivation (requests accept different numbers of tokens, so their
// caches must be re-synchronised) per the EXSPEC/EQSPEC abstract.  For
// k = 0..a the row at slot P + path[k] moves to slot P + k.  The path is
// strictly increasing with path[0] = 0, so path[k] >= k: a source can only
// be clobbered by the destination of an EARLIER k.  Each CTA therefore
// moves the rows in chunks of increasing k and, inside a chunk, reads every
// source into shared memory before writing any destination.  A later chunk
// never reads a slot an earlier chunk wrote (its sources are >= its own k,
// which exceeds every earlier destination).
//
// Grid: (request, K-or-V, KV-head group).  A row of one KV head is D bf16
// (128 or 256 bytes) moved as 16-byte vectors.
#include "walk.cuh"

namespace jsv {

constexpr int kCompactThreads = 256;
constexpr int kCompactChunk = 64;        // rows per chunk
constexpr int kHeadsPerCta = 2;

// Page entries of the tree's slots P .. P + n - 1 (pages P/16 .. (P+n-1)/16),
// staged by the validation pass so that the move needs no page-table loads.
constexpr int kTreePages = 40;           // (n - 1)/16 + 2 for n <= 512

// Moves rows k = 0..acc (slot P + path[k] -> slot P + k) of KV heads
// [h0, h0 + heads) of one cache, in chunks of increasing k; inside a chunk
// every source is read into shared memory before any destination is written.
// `s_pages` holds the checked entries of the tree's pages from page pg0 on.
// Every thread of the block calls it.
__device__ void compact_rows(const BatchArgs &a, const Request &r, const int32_t *pathrow, int acc,
                             uint16_t *cache, int h0, int heads, uint4 *stage, int *s_src, int *s_dst,
                             const int32_t *s_pages, int pg0) {
    const int vec_per_head = a.D / 8;
    const int vec_per_row = heads * vec_per_head;
    const long long cache_elems = (long long)a.num_pages * a.page_size * a.Hkv * a.D;
    auto phys = [&](int slot) { return s_pages[slot / a.page_size - pg0] * a.page_size + slot % a.page_size; };
    for (int k0 = 0; k0 <= acc; k0 += kCompactChunk) {
        const int rows = min(kCompactChunk, acc + 1 - k0);
        for (int i = threadIdx.x; i < rows; i += blockDim.x) {
            s_src[i] = phys(r.P + pathrow[k0 + i]);
            s_dst[i] = phys(r.P + k0 + i);
        }
        __syncthreads();
        for (int e = threadIdx.x; e < rows * vec_per_row; e += blockDim.x) {
            const int i = e / vec_per_row, c = e % vec_per_row;
            const int hh = c / vec_per_head, x = c % vec_per_head;
            if (s_src[i] == s_dst[i]) continue;
            const long long si = ((long long)s_src[i] * a.Hkv + h0 + hh) * a.D + x * 8;
            if (!JSV_IN_BOUNDS(si + 7, cache_elems, a.dev_status) || !JSV_IN_BOUNDS(si, cache_elems, a.dev_status))
                continue;
            stage[e] = *reinterpret_cast<const uint4 *>(cache + si);
        }
        __syncthreads();
        for (int e = threadIdx.x; e < rows * vec_per_row; e += blockDim.x) {
            const int i = e / vec_per_row, c = e % vec_per_row;
            const int hh = c / vec_per_head, x = c % vec_per_head;
            if (s_src[i] == s_dst[i]) continue;
            const long long di = ((long long)s_dst[i] * a.Hkv + h0 + hh) * a.D + x * 8;
            if (!JSV_IN_BOUNDS(di + 7, cache_elems, a.dev_status) || !JSV_IN_BOUNDS(di, cache_elems, a.dev_status))
                continue;
            *reinterpret_cast<uint4 *>(cache + di) = stage[e];
        }
        __syncthreads();
    }
}

// Loads the page entries of the tree's slots (pages P/16 .. (P+n-1)/16) into
// s_pages, spread over the block; returns 1 if any is outside [0, num_pages).
__device__ __forceinline__ int stage_tree_pages(const BatchArgs &a, int b, const Request &r, int32_t *s_pages) {
    const int pg0 = r.P / a.page_size, pg1 = (r.P + r.n - 1) / a.page_size;
    int bad = 0;
    for (int pg = pg0 + threadIdx.x; pg <= pg1; pg += blockDim.x) {
        const long long pi = (long long)b * a.max_pages_per_req + pg;
        const int page = JSV_IN_BOUNDS(pi, (long long)a.B * a.max_pages_per_req, a.dev_status) ? a.page_table[pi] : -1;
        if (page < 0 || page >= a.num_pages) bad = 1;
        s_pages[pg - pg0] = page;
    }
    return bad;
}

__global__ void __launch_bounds__(kCompactThreads)
kv_compact_kernel(BatchArgs a, uint16_t *__restrict__ k_cache, uint16_t *__restrict__ v_cache,
                  const int32_t *__restrict__ path, int max_path,
                  const int32_t *__restrict__ accept_len, int32_t *__restrict__ new_len) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    extern __shared__ uint4 stage[];      // [kCompactChunk][heads][D/8]
    __shared__ int s_src[kCompactChunk], s_dst[kCompactChunk];
    __shared__ int32_t s_pages[kTreePages];
    const int b = blockIdx.x;
    uint16_t *cache = blockIdx.y == 0 ? k_cache : v_cache;
    const int h0 = blockIdx.z * kHeadsPerCta;
    const int heads = min(kHeadsPerCta, a.Hkv - h0);

    // validation, spread over the block: request descriptors, accept length,
    // a strictly increasing path from the root, and every page the move touches
    Request r;
    const bool req_ok = load_request(a, b, r);
    const int acc = req_ok ? accept_len[b] : 0;
    int bad = !req_ok || acc < 0 || acc >= r.n || acc + 1 > max_path;
    const int32_t *row = path + (size_t)b * max_path;
    const int pg0 = req_ok ? r.P / a.page_size : 0;
    if (!bad) {
        for (int k = threadIdx.x; k <= acc; k += blockDim.x) {
            const int pk = row[k];
            if (k == 0 ? pk != 0 : (pk <= row[k - 1] || pk >= r.n)) bad = 1;
        }
        bad |= stage_tree_pages(a, b, r, s_pages);
    }
    bad = __syncthreads_or(bad);
    if (bad) {
        if (threadIdx.x == 0) flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
        return;
    }
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) new_len[b] = r.P + acc + 1;

    compact_rows(a, r, row, acc, cache, h0, heads, stage, s_src, s_dst, s_pages, pg0);
}

// ---------------------------------------------------------------------------
// The accept walk and the compaction in one launch (same grid as the
// compaction).  Every CTA of a request stages the request's tree arrays and
// walks it (a few hundred nanoseconds, from L2), then moves its own
// (K-or-V, head group) rows; the CTA (b, 0, 0) also writes the path,
// accepted length, bonus token and new length.  The outputs equal those of
// jsv_accept_path followed by jsv_kv_compact, error cases included.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kCompactThreads)
accept_compact_kernel(BatchArgs a, const int32_t *__restrict__ tokens, const int32_t *__restrict__ argmax,
                      int max_path, int32_t *__restrict__ path, int32_t *__restrict__ accept_len,
                      int32_t *__restrict__ bonus, uint16_t *__restrict__ k_cache, uint16_t *__restrict__ v_cache,
                      int32_t *__restrict__ new_len) {
    pdl_allow_dependents();
    extern __shared__ uint4 stage[];      // [kCompactChunk][heads][D/8]
    __shared__ int s_src[kCompactChunk], s_dst[kCompactChunk];
    __shared__ int32_t s_par[kWalkMaxNodes], s_tok[kWalkMaxNodes], s_arg[kWalkMaxNodes], s_path[kWalkMaxNodes];
    __shared__ int32_t s_next[kWalkMaxNodes], s_pages[kTreePages];
    __shared__ int s_len, s_last;
    const int b = blockIdx.x;
    const bool writer = blockIdx.y == 0 && blockIdx.z == 0;
    uint16_t *cache = blockIdx.y == 0 ? k_cache : v_cache;
    const int h0 = blockIdx.z * kHeadsPerCta;
    const int heads = min(kHeadsPerCta, a.Hkv - h0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t *row = path + (size_t)b * max_path;

    // Every read comes after the wait for the previous launch (the LM head),
    // the request's geometry included: a caller may pass the previous step's
    // new_len back as prefix_len, and under programmatic dependent launch
    // that step's compaction can still be running while this kernel starts.
    pdl_wait_predecessor();
    Request r;
    const bool req_ok = load_request(a, b, r) && r.n <= kWalkMaxNodes;
    int par_bad = 0, bad = 0;
    const int pg0 = req_ok ? r.P / a.page_size : 0;
    if (req_ok) bad = stage_tree_pages(a, b, r, s_pages);   // every page the move touches must be mapped
    if (req_ok) {
        for (int j = threadIdx.x; j < r.n; j += blockDim.x) {
            const int p = a.parent[r.base + j];
            s_par[j] = p;
            s_tok[j] = tokens[r.base + j];
            s_arg[j] = argmax[r.base + j];
            par_bad |= (j == 0) ? (p != -1) : (p < 0 || p >= j);
        }
    }
    par_bad = __syncthreads_or(par_bad);
    if (!req_ok || par_bad) {
        // the walk's output for an unusable request: the root alone
        if (writer) {
            for (int k = threadIdx.x; k < max_path; k += blockDim.x) row[k] = k == 0 ? 0 : -1;
            if (threadIdx.x == 0) {
                accept_len[b] = 0;
                bonus[b] = -1;
            }
        }
        if (par_bad && threadIdx.x == 0) flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
        if (!req_ok) return;                     // nothing to move (the compaction skips it too)
        if (threadIdx.x == 0) {
            s_path[0] = 0;
            s_len = 1;
        }
    } else {
        if (warp == 0) {
            int last = 0;
            bool cut = false;
            const int len = greedy_walk_warp(s_par, s_tok, s_arg, s_next, r.n, max_path, s_path, lane, last, cut);
            if (lane == 0) {
                s_path[0] = 0;
                s_len = len;
                s_last = last;
                if (cut) flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
            }
        }
        __syncthreads();
        if (writer) {
            for (int k = threadIdx.x; k < max_path; k += blockDim.x) row[k] = k < s_len ? s_path[k] : -1;
            if (threadIdx.x == 0) {
                accept_len[b] = s_len - 1;
                bonus[b] = s_arg[s_last];
            }
        }
    }
    __syncthreads();
    const int acc = s_len - 1;

    bad = __syncthreads_or(bad);
    if (bad) {
        if (threadIdx.x == 0) flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
        return;
    }
    if (threadIdx.x == 0 && writer) new_len[b] = r.P + acc + 1;

    compact_rows(a, r, s_path, acc, cache, h0, heads, stage, s_src, s_dst, s_pages, pg0);
}

cudaError_t launch_kv_compact(const BatchArgs &a, uint16_t *k_cache, uint16_t *v_cache,
                              const int32_t *path, int max_path, const int32_t *accept_len,
                              int32_t *new_len, cudaStream_t st) {
    dim3 grid(a.B, 2, (a.Hkv + kHeadsPerCta - 1) / kHeadsPerCta);
    size_t smem = (size_t)kCompactChunk * kHeadsPerCta * (a.D / 8) * sizeof(uint4);
    static PerDeviceOnce carve;
    cudaError_t e = prefer_max_shared(kv_compact_kernel, carve);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kv_compact_kernel, grid, dim3(kCompactThreads), smem, st, a, k_cache, v_cache, path,
                               max_path, accept_len, new_len);
    count_launches(1);
    return e;
}

cudaError_t launch_accept_compact(const BatchArgs &a, const int32_t *tokens, const int32_t *argmax, int max_path,
                                  int32_t *path, int32_t *accept_len, int32_t *bonus, uint16_t *k_cache,
                                  uint16_t *v_cache, int32_t *new_len, cudaStream_t st) {
    dim3 grid(a.B, 2, (a.Hkv + kHeadsPerCta - 1) / kHeadsPerCta);
    size_t smem = (size_t)kCompactChunk * kHeadsPerCta * (a.D / 8) * sizeof(uint4);
    static PerDeviceOnce carve;
    cudaError_t e = prefer_max_shared(accept_compact_kernel, carve);
    if (e != cudaSuccess) return e;
    e = launch_pdl(accept_compact_kernel, grid, dim3(kCompactThreads), smem, st, a, tokens, argmax, max_path, path,
                   accept_len, bonus, k_cache, v_cache, new_len);
    count_launches(1);
    return e;
}

}  // namespace jsv
