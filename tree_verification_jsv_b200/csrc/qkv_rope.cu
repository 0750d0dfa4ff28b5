// Tree Q/K/V projection with rotary positions; K/V appended to the paged cache.
//
// The step on the other side of the tree attention (reading of the JetSpec
// README, "JetSpec / Overview" and "Quick Start": one forward pass over the
// tree with a paged KV cache).  For node j of request b:
//     qkv = W_qkv x_j          (rows: Q heads, then K heads, then V heads)
// Q and K heads are rotated at position P_b + depth(j) -- a node sits one
// position after its parent, whatever its index -- with the rotate-half pairs
// (i, i + D/2) and caller-supplied fp32 cos/sin tables; Q goes to q[j], K and
// V to logical slot P_b + j of the request's pages (the slots the tree
// attention reads).
//
// Contraction on tcgen05: W rows are the MMA M dimension (one 128-row tile
// per CTA, i.e. one or two heads), the tree nodes are N (up to 256 per
// group), K = d.  A TMA warp streams 64-wide K-chunks of W and x through a
// ring of shared-memory stages, one thread issues tcgen05.mma into a TMEM
// accumulator, and four epilogue warps read it back.  The rotation pairs row
// r with row r ^ D/2 of the same head, which lives in another warp's TMEM
// lanes, so the epilogue stages each 32-node slice of the tile in shared
// memory, then every thread rotates its row against its partner and writes
// bf16 to q or to the cache.
#include "jsv_internal.cuh"
#include "sm100.cuh"

namespace jsv {

using namespace sm100;

namespace {

constexpr int kQThreads = 192;
constexpr int kQMaxStages = 8;
constexpr int kQTileM = 128;
constexpr int kQKChunk = 64;
constexpr uint32_t kQStageA = kQTileM * 128;
constexpr int kQSmemBudget = 180 * 1024;

struct QkvParams {
    BatchArgs a;
    int d, rows_total, kchunks, group_nodes, box_rows, stages;
    uint32_t stage_bytes;
    const float *cos, *sin;
    int max_pos;
    uint16_t *q, *k_cache, *v_cache;
};

__device__ __forceinline__ uint16_t to_bf16_bits(float f) {
    __nv_bfloat16 h = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&h);
}

__global__ void __launch_bounds__(kQThreads, 1)
qkv_rope_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                const QkvParams p) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t full_bar[kQMaxStages], empty_bar[kQMaxStages], accf_bar, drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int ep_fail;
    __shared__ float tile[32][kQTileM];          // one 32-node slice, column-major by node
    __shared__ int s_pos[256], s_row[256];

    const BatchArgs &a = p.a;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = blockIdx.x * kQTileM;
    const int node0 = blockIdx.y * p.group_nodes;
    const int in_group = min(p.group_nodes, a.total_nodes - node0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accf_bar, 1);
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        ep_fail = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmW);
            prefetch_tensormap(&tmX);
            const uint32_t tx = kQStageA + (uint32_t)p.box_rows * 128;
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int kc = 0; kc < p.kchunks; ++kc) {
                if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh)) {
                    abort_sh = 1;
                    flag_error(a.dev_status, JSV_ERR_TIMEOUT);
                    break;
                }
                uint8_t *sa = smem + (size_t)stage * p.stage_bytes;
                mbar_arrive_expect_tx(&full_bar[stage], tx);
                tma_load_2d(sa, &tmW, &full_bar[stage], kc * kQKChunk, row0);
                tma_load_2d(sa + kQStageA, &tmX, &full_bar[stage], kc * kQKChunk, node0);
                ++issued;
                if (++stage == p.stages) { stage = 0; phase ^= 1; }
            }
            if (abort_sh) {
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
            const uint32_t idn = idesc_bf16_f32(kQTileM, (in_group + 15) & ~15, false, false);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kc = 0; kc < p.kchunks; ++kc) {
                if (!mbar_wait(&full_bar[stage], phase, &abort_sh)) {
                    abort_sh = 1;
                    flag_error(a.dev_status, JSV_ERR_TIMEOUT);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_addr(smem + (size_t)stage * p.stage_bytes);
                const uint32_t sb = sa + kQStageA;
#pragma unroll
                for (int kk = 0; kk < kQKChunk / 16; ++kk)
                    mma_bf16_ss(tmem, desc_kmajor_sw128(sa + kk * 32), desc_kmajor_sw128(sb + kk * 32), idn,
                                (kc | kk) != 0);
                mma_commit(&empty_bar[stage]);
                if (++stage == p.stages) { stage = 0; phase ^= 1; }
            }
            if (ok) mma_commit(&accf_bar);
            int zero = 0;
            mma_commit(&drain_bar);
            mbar_wait(&drain_bar, 0, (volatile int *)&zero);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int sub = warp & 3;
        const int r = sub * 32 + lane;               // tile row == TMEM lane
        const int et = threadIdx.x - 64;             // 0..127
        const uint32_t lane_addr = (uint32_t)(sub * 32) << 16;
        // where each node of the group goes: request, position, physical cache row
        for (int c = et; c < in_group; c += 128) {
            const int t = node0 + c;
            int lo = 0, hi = a.B - 1;                // request of node t (node_offsets is sorted)
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (a.node_offsets[mid] <= t) lo = mid; else hi = mid - 1;
            }
            Request req;
            int pos = -1, row = -1;
            if (load_request(a, lo, req)) {
                int j = t - req.base, dep = 0, steps = 0;
                bool ok = true;
                while (j > 0) {
                    const int pj = a.parent[req.base + j];
                    if (pj < 0 || pj >= j || ++steps > req.n) { ok = false; break; }
                    j = pj;
                    ++dep;
                }
                if (ok && req.P + dep < p.max_pos) {
                    pos = req.P + dep;
                    row = (int)slot_phys_row(a, lo, req.P + (t - req.base));
                } else {
                    flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
                }
            }
            s_pos[c] = pos;
            s_row[c] = row;
        }
        named_barrier(1, 128);

        const int grow = row0 + r;                   // global W row of this thread
        const int qrows = a.Hq * a.D, krows = a.Hkv * a.D;
        const int kind = grow < qrows ? 0 : (grow < qrows + krows ? 1 : 2);   // Q, K, V
        const int hrow = kind == 0 ? grow : (kind == 1 ? grow - qrows : grow - qrows - krows);
        const int head = hrow / a.D, o = hrow % a.D, half = a.D / 2;
        const int partner = r ^ half;
        const bool rvalid = grow < p.rows_total;

        if (!mbar_wait(&accf_bar, 0, &abort_sh)) {
            abort_sh = 1;
            flag_error(a.dev_status, JSV_ERR_TIMEOUT);
            ep_fail = 1;
        }
        named_barrier(1, 128);
        if (!ep_fail) {
            tc_fence_after();
            for (int c0 = 0; c0 < in_group; c0 += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + lane_addr + (uint32_t)c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 32; ++x) tile[x][r] = __uint_as_float(v[x]);
                named_barrier(1, 128);
                if (rvalid) {
                    for (int x = 0; x < 32 && c0 + x < in_group; ++x) {
                        const int c = c0 + x;
                        const int pos = s_pos[c], prow = s_row[c];
                        if (pos < 0 || prow < 0) continue;
                        float val = tile[x][r];
                        if (kind < 2) {
                            const int i = o % half;
                            const float cs = p.cos[(size_t)pos * half + i], sn = p.sin[(size_t)pos * half + i];
                            const float pv = tile[x][partner];
                            val = o < half ? fmaf(val, cs, -pv * sn) : fmaf(val, cs, pv * sn);
                        }
                        const int t = node0 + c;
                        const uint16_t hb = to_bf16_bits(val);
                        if (kind == 0) p.q[((size_t)t * a.Hq + head) * a.D + o] = hb;
                        else if (kind == 1) p.k_cache[((size_t)prow * a.Hkv + head) * a.D + o] = hb;
                        else p.v_cache[((size_t)prow * a.Hkv + head) * a.D + o] = hb;
                    }
                }
                named_barrier(1, 128);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace

cudaError_t launch_tree_qkv_rope(const BatchArgs &a, const uint16_t *x, const uint16_t *w_qkv, int d,
                                 const float *rope_cos, const float *rope_sin, int max_pos, uint16_t *q,
                                 uint16_t *k_cache, uint16_t *v_cache, cudaStream_t st) {
    QkvParams p;
    p.a = a;
    p.d = d;
    p.rows_total = (a.Hq + 2 * a.Hkv) * a.D;
    p.kchunks = d / kQKChunk;
    p.group_nodes = a.total_nodes <= 256 ? ((a.total_nodes + 15) & ~15) : 256;
    p.box_rows = p.group_nodes;
    p.stage_bytes = kQStageA + (uint32_t)p.box_rows * 128;
    p.stages = kQSmemBudget / (int)p.stage_bytes;
    if (p.stages > kQMaxStages) p.stages = kQMaxStages;
    p.cos = rope_cos;
    p.sin = rope_sin;
    p.max_pos = max_pos;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;

    CUtensorMap tmW, tmX;
    if (!encode_tensor_map_2d(&tmW, w_qkv, (uint64_t)d, (uint64_t)p.rows_total, (uint64_t)d * 2, kQKChunk, kQTileM))
        return cudaErrorInvalidValue;
    if (!encode_tensor_map_2d(&tmX, x, (uint64_t)d, (uint64_t)a.total_nodes, (uint64_t)d * 2, kQKChunk, p.box_rows))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)p.stages * p.stage_bytes + 1024;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(qkv_rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kQSmemBudget + 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    dim3 grid((p.rows_total + kQTileM - 1) / kQTileM, (a.total_nodes + p.group_nodes - 1) / p.group_nodes);
    cudaError_t e = launch_pdl(qkv_rope_kernel, grid, dim3(kQThreads), smem, st, tmW, tmX, p);
    count_launches(1);
    return e;
}

}  // namespace jsv
