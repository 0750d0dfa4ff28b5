// LM-head projection fused with top-1 argmax, on tcgen05 tensor cores.
//
// JetSpec README, "JetSpec / Overview": the accepted path follows the
// target's own logits, and every reported run is greedy (temperature 0), so
// each node needs only argmax_v <hidden[t], w[v]>.  Logits live in TMEM and
// registers only; they are never written to memory.
//
// Shape of the contraction: logits^T[v][t] = W[v][:] . H[t][:].  The
// vocabulary is the MMA M dimension (128 rows per tile, operand A = W) and
// the tree nodes are the N dimension (operand B = H), so a 64-node tree
// still fills M = 128 and W -- the dominant byte stream -- is read exactly
// once when T <= 512.
//
// Persistent kernel, one CTA per SM, 6 warps:
//   warp 0      TMA producer: W tile (16-row boxes) + H tile per 64-wide K
//               chunk into a ring of shared-memory stages
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, per-column argmax
//               across the 128 vocabulary rows (a transposing butterfly of
//               64-bit keys), then one atomicMax per node
// Each CTA owns a contiguous, balanced vocabulary range [V*c/G, V*(c+1)/G)
// and walks it in 128-row tiles; the ragged last tile of a range loads only
// the 16-row boxes it needs, so no SM gets a whole extra tile of bytes.
// With T <= 256 nodes two accumulators alternate in TMEM so the epilogue of
// one tile overlaps the main loop of the next; larger trees are processed in
// groups of 512 nodes (two N = 256 MMAs per K step, one accumulator).
//
// Cross-CTA reduction: a 64-bit key per node whose high word is the fp32
// value mapped to an order-preserving unsigned integer and whose low word is
// ~index; atomicMax keeps the largest value and, among equal values, the
// smallest index.  The last CTA to finish (a counter in the workspace) writes
// every node's argmax and maximum.
#include "jsv_internal.cuh"
#include "sm100.cuh"

namespace jsv {

using namespace sm100;

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

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
    return a > b ? a : b;
}


constexpr int kMaxStages = 8;
constexpr int kTileM = 128;                    // MMA M (one sub-tile)
constexpr int kBoxRowsW = 16;
constexpr int kKChunk = 64;                    // bf16 elements per 128-B swizzle line
constexpr uint32_t kSubA = kTileM * 128;       // 16 KB: one sub-tile's K-chunk
constexpr int kSmemBudget = 200 * 1024;        // ring of stages (dynamic smem)

// An item is kSub 128-row vocabulary sub-tiles x one node group; the sub-tiles
// share each K-chunk of the node tile.  One sub-tile suits trees of up to 256
// nodes (W streaming dominates); two halve the node-tile traffic for larger
// trees, where the tensor pipe dominates.
template <int kSub>
struct LmShape {
    static constexpr int kEpiWarps = 4 * kSub;     // kSub epilogue warps per TMEM subpartition
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kItemRows = kTileM * kSub;
    static constexpr uint32_t kStageA = kSubA * kSub;
};

struct LmParams {
    int T, d, V;
    int kchunks;       // d / 64
    int ngroups;       // node groups
    int group_nodes;   // nodes per group (<= 256)
    int box_rows;      // H box height (= MMA N of a full group)
    int sub_stride;    // TMEM columns between the two sub-tile accumulators
    int n_acc;         // accumulator sets in TMEM (2 = double buffered, 1)
    int stages;
    uint32_t stage_bytes;
    unsigned long long *keys;
    unsigned int *done;        // CTAs finished (zeroed with the keys before the launch)
    int32_t *argmax;
    float *max_logit;
    int32_t *status;
};

__device__ __forceinline__ void set_abort(volatile int *abort, int32_t *status) {
    *abort = 1;
    if (status) atomicCAS(status, 0, JSV_ERR_TIMEOUT);
}

template <int kSubTiles>
__global__ void __launch_bounds__(LmShape<kSubTiles>::kThreads, 1)
lmhead_argmax_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmW16,
                        const __grid_constant__ CUtensorMap tmH, const LmParams p) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    constexpr int kEpiWarps = LmShape<kSubTiles>::kEpiWarps;
    constexpr int kItemRows = LmShape<kSubTiles>::kItemRows;
    constexpr uint32_t kStageA = LmShape<kSubTiles>::kStageA;
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int ep_fail;
    __shared__ unsigned long long red[kEpiWarps][256];

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const int r0 = (int)((long long)p.V * cta / G), r1 = (int)((long long)p.V * (cta + 1) / G);
    const int ntiles = (r1 - r0 + kItemRows - 1) / kItemRows;
    const int items = ntiles * p.ngroups;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accf_bar[a], 1);
            mbar_init(&acce_bar[a], kEpiWarps);
        }
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        ep_fail = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmW);
        prefetch_tensormap(&tmW16);
        prefetch_tensormap(&tmH);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_h = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int it = 0; it < items && !abort_sh; ++it) {
                const int vt = it / p.ngroups, g = it % p.ngroups;
                const int row0 = r0 + vt * kItemRows;
                int rows[kSubTiles];
                uint32_t tx = (uint32_t)p.box_rows * 128;
#pragma unroll
                for (int s = 0; s < kSubTiles; ++s) {
                    rows[s] = max(0, min(kTileM, r1 - (row0 + s * kTileM)));
                    tx += rows[s] == kTileM ? kSubA : (uint32_t)((rows[s] + kBoxRowsW - 1) / kBoxRowsW) * (kBoxRowsW * 128);
                }
                const int node0 = g * p.group_nodes;
                bool ok = true;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh)) {
                        set_abort(&abort_sh, p.status);
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + (size_t)stage * p.stage_bytes;
                    uint8_t *sb = sa + kStageA;
                    mbar_arrive_expect_tx(&full_bar[stage], tx);
#pragma unroll
                    for (int s = 0; s < kSubTiles; ++s) {
                        const int rs = row0 + s * kTileM;
                        if (rows[s] == kTileM) {
                            tma_load_2d_hint(sa + s * kSubA, &tmW, &full_bar[stage], kc * kKChunk, rs, pol_w);
                        } else {
                            for (int bx = 0; bx * kBoxRowsW < rows[s]; ++bx)
                                tma_load_2d_hint(sa + s * kSubA + bx * (kBoxRowsW * 128), &tmW16, &full_bar[stage],
                                                 kc * kKChunk, rs + bx * kBoxRowsW, pol_w);
                        }
                    }
                    tma_load_2d_hint(sb, &tmH, &full_bar[stage], kc * kKChunk, node0, pol_h);
                    ++issued;
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (abort_sh) {
                // let every load still in flight land before the CTA exits
                int zero = 0;
                const long long back = issued < p.stages ? issued : p.stages;
                int s = stage;
                uint32_t ph = phase;
                for (long long i = 0; i < back; ++i) {
                    if (s == 0) { s = p.stages; ph ^= 1; }
                    --s;
                    mbar_wait(&full_bar[s], ph, (volatile int *)&zero);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int it = 0; it < items && !abort_sh; ++it) {
                const int acc = it % p.n_acc;
                const uint32_t use = (uint32_t)(it / p.n_acc);
                if (!mbar_wait(&acce_bar[acc], (use & 1) ^ 1, &abort_sh)) {
                    set_abort(&abort_sh, p.status);
                    break;
                }
                tc_fence_after();
                const int vt = it / p.ngroups, g = it % p.ngroups;
                const int row0 = r0 + vt * kItemRows;
                const bool sub1 = kSubTiles > 1 && r1 - (row0 + kTileM) > 0;   // second sub-tile has rows
                const int in_group = min(p.group_nodes, p.T - g * p.group_nodes);
                const uint32_t idn = idesc_bf16_f32(kTileM, (in_group + 15) & ~15, false, false);
                const uint32_t d0 = tmem + (uint32_t)acc * 256u;
                bool ok = true;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&full_bar[stage], phase, &abort_sh)) {
                        set_abort(&abort_sh, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + (size_t)stage * p.stage_bytes);
                    const uint32_t sb = sa + kStageA;
#pragma unroll
                    for (int kk = 0; kk < kKChunk / 16; ++kk) {
                        const uint32_t accum = (kc | kk) != 0;
                        const uint64_t bdesc = desc_kmajor_sw128(sb + kk * 32);
                        mma_bf16_ss(d0, desc_kmajor_sw128(sa + kk * 32), bdesc, idn, accum);
                        if (kSubTiles > 1 && sub1)
                            mma_bf16_ss(d0 + (uint32_t)p.sub_stride, desc_kmajor_sw128(sa + kSubA + kk * 32), bdesc,
                                        idn, accum);
                    }
                    mma_commit(&empty_bar[stage]);
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&accf_bar[acc]);
            }
            // every MMA issued above has finished before TMEM is released
            int zero = 0;
            mma_commit(&drain_bar);
            mbar_wait(&drain_bar, 0, (volatile int *)&zero);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;                     // 0..7
        const int subt = ew >> 2;                    // vocabulary sub-tile this warp reads
        const int sub = warp & 3;                    // TMEM lanes this warp may access
        const uint32_t lane_addr = (uint32_t)(sub * 32) << 16;
        const int et = threadIdx.x - 64;             // 0..255
        for (int it = 0; it < items; ++it) {
            const int acc = it % p.n_acc;
            const uint32_t use = (uint32_t)(it / p.n_acc);
            if (!mbar_wait(&accf_bar[acc], use & 1, &abort_sh)) {
                set_abort(&abort_sh, p.status);
                ep_fail = 1;
            }
            named_barrier(1, 32 * kEpiWarps);
            if (ep_fail) break;
            tc_fence_after();
            const int vt = it / p.ngroups, g = it % p.ngroups;
            const int v = r0 + vt * kItemRows + subt * kTileM + sub * 32 + lane;
            const bool vvalid = v < r1;
            const int node0 = g * p.group_nodes;
            const int in_group = min(p.group_nodes, p.T - node0);
            const int ncols = (in_group + 31) & ~31;
            const uint32_t base = tmem + lane_addr + (uint32_t)acc * 256u + (uint32_t)(subt * p.sub_stride);
            for (int c0 = 0; c0 < ncols; c0 += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(base + (uint32_t)c0, r);
                tmem_ld_wait();
                unsigned long long x[32];
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    x[j] = (vvalid && c0 + j < in_group) ? argmax_key(__uint_as_float(r[j]), v) : 0ull;
                // transposing butterfly: afterwards lane l holds column c0 + l
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                    const bool upper = (lane & o) != 0;
#pragma unroll
                    for (int i = 0; i < o; ++i) {
                        const unsigned long long send = upper ? x[i] : x[i + o];
                        const unsigned long long keep = upper ? x[i + o] : x[i];
                        x[i] = umax64(keep, __shfl_xor_sync(0xffffffffu, send, o));
                    }
                }
                red[ew][c0 + lane] = x[0];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar[acc]);
            named_barrier(1, 32 * kEpiWarps);
            for (int c = et; c < in_group; c += 32 * kEpiWarps) {
                unsigned long long k = red[0][c];
#pragma unroll
                for (int w = 1; w < kEpiWarps; ++w) k = umax64(k, red[w][c]);
                if (k) atomicMax(&p.keys[node0 + c], k);
            }
            named_barrier(1, 32 * kEpiWarps);
        }
    }

    tc_fence_before();
    __threadfence();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    // the last CTA to finish turns every node's key into its argmax
    __shared__ int is_last;
    if (threadIdx.x == 0) is_last = atomicAdd(p.done, 1u) == (unsigned)(gridDim.x - 1);
    __syncthreads();
    if (is_last) {
        __threadfence();
        for (int t = threadIdx.x; t < p.T; t += blockDim.x) {
            const unsigned long long k = atomicAdd(&p.keys[t], 0ull);
            p.argmax[t] = (int32_t)(~(uint32_t)(k & 0xffffffffull));
            if (p.max_logit) p.max_logit[t] = key_value(k);
        }
    }
}

size_t lmhead_workspace_bytes(int T, int d, int V) {
    (void)d; (void)V;
    return (size_t)T * sizeof(unsigned long long) + sizeof(unsigned long long);   // keys + done counter
}

cudaError_t launch_lmhead_argmax(const uint16_t *hidden, const uint16_t *w, int T, int d, int V,
                                 int32_t *argmax, float *max_logit, void *ws, cudaStream_t st) {
    int32_t *status = nullptr;
    auto *keys = static_cast<unsigned long long *>(ws);
    const int sub = T <= 256 ? 1 : 2;
    LmParams p;
    p.T = T; p.d = d; p.V = V;
    p.kchunks = d / kKChunk;
    if (sub == 1) {
        // one 128-row accumulator per item, two items in flight in TMEM
        p.group_nodes = (T + 15) & ~15;
        p.sub_stride = 0;
        p.n_acc = 2;
    } else {
        // two 128-row accumulators of up to 256 nodes fill TMEM: one item in flight
        p.group_nodes = 256;
        p.sub_stride = 256;
        p.n_acc = 1;
    }
    p.box_rows = p.group_nodes;
    p.ngroups = (T + p.group_nodes - 1) / p.group_nodes;
    p.stage_bytes = kSubA * sub + (uint32_t)p.box_rows * 128;
    p.stages = kSmemBudget / (int)p.stage_bytes;
    if (p.stages > kMaxStages) p.stages = kMaxStages;
    p.keys = keys;
    p.done = reinterpret_cast<unsigned int *>(keys + T);
    p.argmax = argmax;
    p.max_logit = max_logit;
    p.status = status;

    CUtensorMap tmW, tmW16, tmH;
    if (!encode_tensor_map_2d(&tmW, w, (uint64_t)d, (uint64_t)V, (uint64_t)d * 2, kKChunk, kTileM))
        return cudaErrorInvalidValue;
    if (!encode_tensor_map_2d(&tmW16, w, (uint64_t)d, (uint64_t)V, (uint64_t)d * 2, kKChunk, kBoxRowsW))
        return cudaErrorInvalidValue;
    if (!encode_tensor_map_2d(&tmH, hidden, (uint64_t)d, (uint64_t)T, (uint64_t)d * 2, kKChunk, p.box_rows))
        return cudaErrorInvalidValue;

    const size_t smem = (size_t)p.stages * p.stage_bytes + 1024;
    static bool attr_set[64][2] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev][sub - 1]) {
        cudaError_t e = sub == 1 ? cudaFuncSetAttribute(lmhead_argmax_tc_kernel<1>,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget + 1024)
                                 : cudaFuncSetAttribute(lmhead_argmax_tc_kernel<2>,
                                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget + 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev][sub - 1] = true;
    }
    cudaError_t e = cudaMemsetAsync(keys, 0, lmhead_workspace_bytes(T, d, V), st);
    if (e != cudaSuccess) return e;
    const int item_rows = kTileM * sub;
    const int tiles = (V + item_rows - 1) / item_rows;
    int grid = device_sm_count();
    if (grid <= 0) return cudaErrorInvalidDevice;
    if (grid > tiles) grid = tiles;
    if (sub == 1)
        e = launch_pdl(lmhead_argmax_tc_kernel<1>, dim3(grid), dim3(LmShape<1>::kThreads), smem, st, tmW, tmW16, tmH, p);
    else
        e = launch_pdl(lmhead_argmax_tc_kernel<2>, dim3(grid), dim3(LmShape<2>::kThreads), smem, st, tmW, tmW16, tmH, p);
    count_launches(1);
    return e;
}

}  // namespace jsv
