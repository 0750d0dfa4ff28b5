// Tree-causal attention over a paged KV prefix, split-KV.
//
// JetSpec README, "JetSpec / Overview": the whole draft tree is verified in
// one forward pass under a tree-causal mask.  Node i of request b attends to
// prefix slots [0, P) and to slot P + j for every ancestor-or-self j of i.
// The prefix is cut into S splits processed by separate CTAs; the tree part
// rides with the last split; a combine pass merges the (max, sum, output)
// partials with the usual log-sum-exp rescaling.
//
// SIMT version: one warp per (node, query head, split); each lane owns D/32
// output dimensions.
#include "jsv_internal.cuh"

#include <math.h>

namespace jsv {

constexpr int kAttnWarps = 8;

static int attention_splits(const BatchArgs &a) {
    int s = (a.max_prefix + 511) / 512;
    return s < 1 ? 1 : (s > 16 ? 16 : s);
}

size_t attention_workspace_bytes(const BatchArgs &a) {
    const size_t rows = (size_t)a.total_nodes * a.Hq;
    return (size_t)attention_splits(a) * rows * ((size_t)a.D + 2) * sizeof(float);
}

// Ancestor-or-self bitset of request-local node i: lane w holds bits
// [32w, 32w + 32).  Returns false if the parent chain is malformed.
__device__ __forceinline__ bool ancestor_bits(const BatchArgs &a, const Request &r, int i,
                                              int lane, unsigned &bits) {
    bits = 0;
    int j = i, steps = 0;
    while (j != -1) {
        if (steps++ > r.n) return false;
        if ((j >> 5) == lane) bits |= 1u << (j & 31);
        const int p = a.parent[r.base + j];
        if (j == 0 ? p != -1 : (p < 0 || p >= j)) return false;
        j = p;
    }
    return true;
}

template <int D>
__global__ void __launch_bounds__(kAttnWarps * 32)
tree_attention_simt_kernel(BatchArgs a, const uint16_t *__restrict__ q,
                           const uint16_t *__restrict__ kc, const uint16_t *__restrict__ vc,
                           float scale_log2, int S, float *__restrict__ ws_o,
                           float *__restrict__ ws_ml) {
    constexpr int DPL = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.z / a.Hkv, g = blockIdx.z % a.Hkv;
    const int G = a.Hq / a.Hkv;
    const int rloc = blockIdx.x * kAttnWarps + warp;
    const int split = blockIdx.y;
    Request r;
    if (!load_request(a, b, r)) return;
    if (rloc >= r.n * G) return;
    const int i = rloc / G, h = g * G + rloc % G, t = r.base + i;
    unsigned anc;
    if (!ancestor_bits(a, r, i, lane, anc)) {
        if (lane == 0) flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
        return;
    }
    float qv[DPL];
    const uint16_t *qp = q + ((size_t)t * a.Hq + h) * D + lane * DPL;
#pragma unroll
    for (int x = 0; x < DPL; ++x) qv[x] = bf16_bits_to_float(qp[x]) * scale_log2;

    float m = -INFINITY, l = 0.f, o[DPL];
#pragma unroll
    for (int x = 0; x < DPL; ++x) o[x] = 0.f;

    auto visit = [&](int slot) {
        const long long row = slot_phys_row(a, b, slot);
        if (row < 0) return;
        const size_t off = ((size_t)row * a.Hkv + g) * D + lane * DPL;
        float part = 0.f;
#pragma unroll
        for (int x = 0; x < DPL; ++x) part = fmaf(qv[x], bf16_bits_to_float(kc[off + x]), part);
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) part += __shfl_xor_sync(0xffffffffu, part, sh);
        const float mn = fmaxf(m, part);
        const float c = exp2f(m - mn), p = exp2f(part - mn);
        l = l * c + p;
#pragma unroll
        for (int x = 0; x < DPL; ++x) o[x] = fmaf(p, bf16_bits_to_float(vc[off + x]), o[x] * c);
        m = mn;
    };

    const int lo = (int)((long long)r.P * split / S), hi = (int)((long long)r.P * (split + 1) / S);
    for (int s = lo; s < hi; ++s) visit(s);
    if (split == S - 1) {
        for (int j = 0; j < r.n; ++j) {
            const unsigned w = __shfl_sync(0xffffffffu, anc, j >> 5);
            if ((w >> (j & 31)) & 1u) visit(r.P + j);
        }
    }
    const size_t row_id = (size_t)t * a.Hq + h;
    const size_t rows = (size_t)a.total_nodes * a.Hq;
    float *po = ws_o + ((size_t)split * rows + row_id) * D + lane * DPL;
#pragma unroll
    for (int x = 0; x < DPL; ++x) po[x] = o[x];
    if (lane == 0) {
        ws_ml[((size_t)split * rows + row_id) * 2 + 0] = m;
        ws_ml[((size_t)split * rows + row_id) * 2 + 1] = l;
    }
}

template <int D>
__global__ void __launch_bounds__(kAttnWarps * 32)
tree_attention_combine_kernel(BatchArgs a, int S, const float *__restrict__ ws_o,
                              const float *__restrict__ ws_ml, uint16_t *__restrict__ out) {
    constexpr int DPL = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.z / a.Hkv, g = blockIdx.z % a.Hkv;
    const int G = a.Hq / a.Hkv;
    const int rloc = blockIdx.x * kAttnWarps + warp;
    Request r;
    if (!load_request(a, b, r)) return;
    if (rloc >= r.n * G) return;
    const int i = rloc / G, h = g * G + rloc % G, t = r.base + i;
    const size_t row_id = (size_t)t * a.Hq + h;
    const size_t rows = (size_t)a.total_nodes * a.Hq;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) {
        const float l = ws_ml[((size_t)s * rows + row_id) * 2 + 1];
        if (l > 0.f) M = fmaxf(M, ws_ml[((size_t)s * rows + row_id) * 2]);
    }
    float L = 0.f, o[DPL];
#pragma unroll
    for (int x = 0; x < DPL; ++x) o[x] = 0.f;
    for (int s = 0; s < S; ++s) {
        const float l = ws_ml[((size_t)s * rows + row_id) * 2 + 1];
        if (!(l > 0.f)) continue;
        const float c = exp2f(ws_ml[((size_t)s * rows + row_id) * 2] - M);
        L = fmaf(l, c, L);
        const float *po = ws_o + ((size_t)s * rows + row_id) * D + lane * DPL;
#pragma unroll
        for (int x = 0; x < DPL; ++x) o[x] = fmaf(c, po[x], o[x]);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    uint16_t *op = out + row_id * D + lane * DPL;
#pragma unroll
    for (int x = 0; x < DPL; ++x) {
        __nv_bfloat16 hb = __float2bfloat16_rn(o[x] * inv);
        op[x] = *reinterpret_cast<uint16_t *>(&hb);
    }
}

cudaError_t launch_tree_attention(const BatchArgs &a, const uint16_t *q, const uint16_t *k_cache,
                                  const uint16_t *v_cache, float scale, uint16_t *out, void *ws,
                                  cudaStream_t st) {
    const int S = attention_splits(a);
    const int G = a.Hq / a.Hkv;
    const size_t rows = (size_t)a.total_nodes * a.Hq;
    float *ws_o = static_cast<float *>(ws);
    float *ws_ml = ws_o + (size_t)S * rows * a.D;
    const float scale_log2 = scale * 1.4426950408889634f;
    dim3 grid((a.max_nodes * G + kAttnWarps - 1) / kAttnWarps, S, a.B * a.Hkv);
    dim3 cgrid(grid.x, 1, grid.z);
    if (a.D == 128) {
        tree_attention_simt_kernel<128><<<grid, kAttnWarps * 32, 0, st>>>(a, q, k_cache, v_cache,
                                                                          scale_log2, S, ws_o, ws_ml);
        tree_attention_combine_kernel<128><<<cgrid, kAttnWarps * 32, 0, st>>>(a, S, ws_o, ws_ml, out);
    } else {
        tree_attention_simt_kernel<64><<<grid, kAttnWarps * 32, 0, st>>>(a, q, k_cache, v_cache,
                                                                         scale_log2, S, ws_o, ws_ml);
        tree_attention_combine_kernel<64><<<cgrid, kAttnWarps * 32, 0, st>>>(a, S, ws_o, ws_ml, out);
    }
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace jsv
