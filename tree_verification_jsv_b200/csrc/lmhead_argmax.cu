// LM-head projection fused with top-1 argmax.
//
// JetSpec README, "JetSpec / Overview": the accepted path follows the
// target's own logits; every reported run is greedy (temperature 0), so
// each node needs only argmax_v <hidden[t], w[v]>.  Logits are reduced in
// registers / shared memory and never written to memory.
//
// Cross-CTA reduction: each CTA folds its best (value, index) per node into
// one 64-bit key with atomicMax.  The high word is the fp32 value mapped to
// an order-preserving unsigned integer, the low word is ~index, so the
// maximum key carries the largest value and, among equal values, the
// smallest index.
#include "jsv_internal.cuh"

namespace jsv {

__device__ __forceinline__ unsigned long long argmax_key(float f, int v) {
    if (f == 0.0f) f = 0.0f;                       // -0 and +0 compare equal
    const uint32_t u = __float_as_uint(f);
    const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)o << 32) | (uint32_t)(~(uint32_t)v);
}

__device__ __forceinline__ float key_value(unsigned long long k) {
    const uint32_t o = (uint32_t)(k >> 32);
    const uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
    return __uint_as_float(u);
}

__global__ void argmax_finalize_kernel(const unsigned long long *__restrict__ keys, int T,
                                       int32_t *__restrict__ argmax, float *__restrict__ max_logit) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const unsigned long long k = keys[t];
    argmax[t] = (int32_t)(~(uint32_t)(k & 0xffffffffull));
    if (max_logit) max_logit[t] = key_value(k);
}

// ---------------------------------------------------------------------------
// SIMT tile: 64 vocabulary rows x 64 nodes per CTA, 4x4 outputs per thread.
// ---------------------------------------------------------------------------
constexpr int kTV = 64, kTT = 64, kTK = 32;

__global__ void __launch_bounds__(256)
lmhead_argmax_simt_kernel(const uint16_t *__restrict__ H, const uint16_t *__restrict__ W,
                          int T, int d, int V, unsigned long long *__restrict__ keys) {
    __shared__ float Ws[kTK][kTV + 4];
    __shared__ float Hs[kTK][kTT + 4];
    __shared__ unsigned long long red[16][kTT];
    const int v0 = blockIdx.x * kTV, t0 = blockIdx.y * kTT;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < d; k0 += kTK) {
        for (int e = threadIdx.x; e < kTV * kTK; e += 256) {
            const int r = e / kTK, kk = e % kTK, v = v0 + r;
            Ws[kk][r] = v < V ? bf16_bits_to_float(W[(size_t)v * d + k0 + kk]) : 0.f;
        }
        for (int e = threadIdx.x; e < kTT * kTK; e += 256) {
            const int r = e / kTK, kk = e % kTK, t = t0 + r;
            Hs[kk][r] = t < T ? bf16_bits_to_float(H[(size_t)t * d + k0 + kk]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kTK; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = Ws[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = Hs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        unsigned long long best = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int v = v0 + ty * 4 + i;
            if (v < V) {
                const unsigned long long k = argmax_key(acc[i][j], v);
                best = k > best ? k : best;
            }
        }
        red[ty][tx * 4 + j] = best;
    }
    __syncthreads();
    if (threadIdx.x < kTT) {
        unsigned long long best = 0;
        for (int y = 0; y < 16; ++y) best = red[y][threadIdx.x] > best ? red[y][threadIdx.x] : best;
        const int t = t0 + threadIdx.x;
        if (t < T && best) atomicMax(&keys[t], best);
    }
}

size_t lmhead_workspace_bytes(int T, int d, int V) {
    (void)d; (void)V;
    return (size_t)T * sizeof(unsigned long long);
}

cudaError_t launch_lmhead_argmax(const uint16_t *hidden, const uint16_t *w, int T, int d, int V,
                                 int32_t *argmax, float *max_logit, void *ws, cudaStream_t st) {
    auto *keys = static_cast<unsigned long long *>(ws);
    cudaError_t e = cudaMemsetAsync(keys, 0, (size_t)T * sizeof(unsigned long long), st);
    if (e != cudaSuccess) return e;
    dim3 grid((V + kTV - 1) / kTV, (T + kTT - 1) / kTT);
    lmhead_argmax_simt_kernel<<<grid, 256, 0, st>>>(hidden, w, T, d, V, keys);
    argmax_finalize_kernel<<<(T + 255) / 256, 256, 0, st>>>(keys, T, argmax, max_logit);
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace jsv
