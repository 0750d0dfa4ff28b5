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
#include "jsv_internal.cuh"

namespace jsv {

constexpr int kCompactThreads = 256;
constexpr int kCompactChunk = 64;        // rows per chunk
constexpr int kHeadsPerCta = 2;

__global__ void __launch_bounds__(kCompactThreads)
kv_compact_kernel(BatchArgs a, uint16_t *__restrict__ k_cache, uint16_t *__restrict__ v_cache,
                  const int32_t *__restrict__ path, int max_path,
                  const int32_t *__restrict__ accept_len, int32_t *__restrict__ new_len) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    extern __shared__ uint4 stage[];      // [kCompactChunk][heads][D/8]
    __shared__ int s_src[kCompactChunk], s_dst[kCompactChunk];
    const int b = blockIdx.x;
    uint16_t *cache = blockIdx.y == 0 ? k_cache : v_cache;
    const int h0 = blockIdx.z * kHeadsPerCta;
    const int heads = min(kHeadsPerCta, a.Hkv - h0);
    const int vec_per_head = a.D / 8;
    const int vec_per_row = heads * vec_per_head;

    // validation, spread over the block: request descriptors, accept length,
    // a strictly increasing path from the root, and every page the move touches
    Request r;
    const bool req_ok = load_request(a, b, r);
    const int acc = req_ok ? accept_len[b] : 0;
    int bad = !req_ok || acc < 0 || acc >= r.n || acc + 1 > max_path;
    const int32_t *row = path + (size_t)b * max_path;
    if (!bad) {
        for (int k = threadIdx.x; k <= acc; k += blockDim.x) {
            const int pk = row[k];
            if (k == 0 ? pk != 0 : (pk <= row[k - 1] || pk >= r.n)) bad = 1;
        }
        const int pg0 = r.P / a.page_size, pg1 = (r.P + r.n - 1) / a.page_size;
        for (int pg = pg0 + threadIdx.x; pg <= pg1; pg += blockDim.x) {
            const int page = a.page_table[(size_t)b * a.max_pages_per_req + pg];
            if (page < 0 || page >= a.num_pages) bad = 1;
        }
    }
    bad = __syncthreads_or(bad);
    if (bad) {
        if (threadIdx.x == 0) flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
        return;
    }
    if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) new_len[b] = r.P + acc + 1;

    for (int k0 = 0; k0 <= acc; k0 += kCompactChunk) {
        const int rows = min(kCompactChunk, acc + 1 - k0);
        for (int i = threadIdx.x; i < rows; i += blockDim.x) {
            s_src[i] = (int)slot_phys_row(a, b, r.P + row[k0 + i]);
            s_dst[i] = (int)slot_phys_row(a, b, r.P + k0 + i);
        }
        __syncthreads();
        for (int e = threadIdx.x; e < rows * vec_per_row; e += blockDim.x) {
            const int i = e / vec_per_row, c = e % vec_per_row;
            const int hh = c / vec_per_head, x = c % vec_per_head;
            if (s_src[i] == s_dst[i]) continue;
            const uint4 *src = reinterpret_cast<const uint4 *>(
                cache + ((size_t)s_src[i] * a.Hkv + h0 + hh) * a.D);
            stage[e] = src[x];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < rows * vec_per_row; e += blockDim.x) {
            const int i = e / vec_per_row, c = e % vec_per_row;
            const int hh = c / vec_per_head, x = c % vec_per_head;
            if (s_src[i] == s_dst[i]) continue;
            uint4 *dst = reinterpret_cast<uint4 *>(cache + ((size_t)s_dst[i] * a.Hkv + h0 + hh) * a.D);
            dst[x] = stage[e];
        }
        __syncthreads();
    }
}

cudaError_t launch_kv_compact(const BatchArgs &a, uint16_t *k_cache, uint16_t *v_cache,
                              const int32_t *path, int max_path, const int32_t *accept_len,
                              int32_t *new_len, cudaStream_t st) {
    dim3 grid(a.B, 2, (a.Hkv + kHeadsPerCta - 1) / kHeadsPerCta);
    size_t smem = (size_t)kCompactChunk * kHeadsPerCta * (a.D / 8) * sizeof(uint4);
    static bool carve[64] = {};
    cudaError_t e = prefer_max_shared(kv_compact_kernel, carve);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kv_compact_kernel, grid, dim3(kCompactThreads), smem, st, a, k_cache, v_cache, path,
                               max_path, accept_len, new_len);
    count_launches(1);
    return e;
}

}  // namespace jsv
