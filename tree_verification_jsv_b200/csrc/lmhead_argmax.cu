// LM-head projection fused with top-1 argmax, on tcgen05 tensor cores.
//
// JetSpec README, "JetSpec / Overview": the accepted path follows the
// target's own logits, and every reported run is greedy (temperature 0), so
// each node needs only argmax_v <hidden[t], w[v]>.  Logits live in TMEM and
// registers only; they are never written to memory.
//
// Shape of the contraction: logits^T[v][t] = W[v][:] . H[t][:].  The
// vocabulary is the MMA M dimension (128 rows per tile, operand A = W) and
// the tree nodes are the N dimension (operand B = H, up to 256 nodes per
// MMA), so a 64-node tree still fills M = 128.
//
// An item is one 128-row vocabulary tile x one group of up to 256 nodes.
// Persistent kernel, one CTA per SM, 6 warps:
//   warp 0      TMA producer: W tile (16-row boxes for a ragged tile) + H
//               tile per 64-wide K chunk into a ring of shared-memory stages
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, per-column argmax
//               across the 128 vocabulary rows (a transposing butterfly of
//               64-bit keys), then one atomicMax per node
// Two accumulators alternate in TMEM, so the epilogue of one item overlaps
// the main loop of the next.
// Work split: with one node group (up to 256 nodes; W, the dominant byte
// stream, is read exactly once) each CTA owns a contiguous, balanced
// vocabulary range [V*c/G, V*(c+1)/G) whose ragged last tile loads only the
// 16-row boxes it needs.  With several node groups the tensor pipe
// dominates: each CTA takes a balanced contiguous range of the (tile, group)
// items, group fastest, so consecutive items reuse the same W tile from L2.
//
// Node groups above 128 (tensor-bound) run on CTA pairs with 2-SM MMAs; see
// the pair kernel below.
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
constexpr int kTileM = 128;                    // MMA M: vocabulary rows of a tile
constexpr int kMaxGroupNodes = 256;            // MMA N: nodes of a group
constexpr int kBoxRowsW = 16;
constexpr int kKChunk = 64;                    // bf16 elements per 128-B swizzle line
constexpr uint32_t kStageA = kTileM * 128;     // 16 KB: a W tile's K-chunk
constexpr int kSmemBudget = 200 * 1024;        // ring of stages (dynamic smem)
constexpr int kEpiWarps = 4;                   // one per TMEM subpartition
constexpr int kLmThreads = 64 + 32 * kEpiWarps;

struct LmParams {
    int T, d, V;
    int kchunks;       // d / 64
    int ngroups;       // node groups
    int group_nodes;   // nodes per group (<= 256): the H box height
    int stages;
    uint32_t stage_bytes;
    unsigned long long *keys;
    unsigned int *done;        // CTAs finished (zeroed with the keys before the launch)
    int32_t *argmax;
    float *max_logit;
    int32_t *status;
};

// The k-th item of a CTA: vocabulary rows [row0, row0 + rows) and node group g.
struct LmItem {
    int row0, rows, g;
};

struct LmWork {
    int r0, r1;        // vocabulary range (one node group)
    int it0;           // first global item (several node groups)
    int items;

    __device__ LmWork(const LmParams &p, int cta, int G) {
        if (p.ngroups == 1) {
            r0 = (int)((long long)p.V * cta / G);
            r1 = (int)((long long)p.V * (cta + 1) / G);
            it0 = 0;
            items = (r1 - r0 + kTileM - 1) / kTileM;
        } else {
            const long long total = (long long)((p.V + kTileM - 1) / kTileM) * p.ngroups;
            r0 = r1 = 0;
            it0 = (int)(total * cta / G);
            items = (int)(total * (cta + 1) / G) - it0;
        }
    }
    __device__ LmItem item(const LmParams &p, int k) const {
        LmItem t;
        if (p.ngroups == 1) {
            t.row0 = r0 + k * kTileM;
            t.rows = min(kTileM, r1 - t.row0);
            t.g = 0;
        } else {
            const int i = it0 + k, vt = i / p.ngroups;
            t.row0 = vt * kTileM;
            t.rows = min(kTileM, p.V - t.row0);
            t.g = i - vt * p.ngroups;
        }
        return t;
    }
};

__device__ __forceinline__ void set_abort(volatile int *abort, int32_t *status) {
    *abort = 1;
    if (status) atomicCAS(status, 0, JSV_ERR_TIMEOUT);
}

__global__ void __launch_bounds__(kLmThreads, 1)
lmhead_argmax_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmW16,
                        const __grid_constant__ CUtensorMap tmH, const LmParams p) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int ep_fail;
    __shared__ unsigned long long red[kEpiWarps][kMaxGroupNodes];

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const LmWork work(p, blockIdx.x, gridDim.x);
    const int items = work.items;

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
            // W is read once with one node group (stream it past L2), several
            // times from L2 with several; H is re-read by every item
            const uint64_t pol_w = p.ngroups == 1 ? policy_evict_first() : policy_evict_normal();
            const uint64_t pol_h = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int it = 0; it < items && !abort_sh; ++it) {
                const LmItem t = work.item(p, it);
                const uint32_t tx = (uint32_t)p.group_nodes * 128 +
                                    (t.rows == kTileM ? kStageA
                                                      : (uint32_t)((t.rows + kBoxRowsW - 1) / kBoxRowsW) * (kBoxRowsW * 128));
                const int node0 = t.g * p.group_nodes;
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
                    if (t.rows == kTileM) {
                        tma_load_2d_hint(sa, &tmW, &full_bar[stage], kc * kKChunk, t.row0, pol_w);
                    } else {
                        for (int bx = 0; bx * kBoxRowsW < t.rows; ++bx)
                            tma_load_2d_hint(sa + bx * (kBoxRowsW * 128), &tmW16, &full_bar[stage], kc * kKChunk,
                                             t.row0 + bx * kBoxRowsW, pol_w);
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
                const int acc = it & 1;
                const uint32_t use = (uint32_t)(it >> 1);
                if (!mbar_wait(&acce_bar[acc], (use & 1) ^ 1, &abort_sh)) {
                    set_abort(&abort_sh, p.status);
                    break;
                }
                tc_fence_after();
                const LmItem t = work.item(p, it);
                const int in_group = min(p.group_nodes, p.T - t.g * p.group_nodes);
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
                    for (int kk = 0; kk < kKChunk / 16; ++kk)
                        mma_bf16_ss(d0, desc_kmajor_sw128(sa + kk * 32), desc_kmajor_sw128(sb + kk * 32), idn,
                                    (kc | kk) != 0);
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
        const int ew = warp - 2;                     // 0..3
        const int sub = warp & 3;                    // TMEM lanes this warp may access
        const uint32_t lane_addr = (uint32_t)(sub * 32) << 16;
        const int et = threadIdx.x - 64;             // 0..127
        for (int it = 0; it < items; ++it) {
            const int acc = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            if (!mbar_wait(&accf_bar[acc], use & 1, &abort_sh)) {
                set_abort(&abort_sh, p.status);
                ep_fail = 1;
            }
            named_barrier(1, 32 * kEpiWarps);
            if (ep_fail) break;
            tc_fence_after();
            const LmItem t = work.item(p, it);
            const int v = t.row0 + sub * 32 + lane;
            const bool vvalid = v < t.row0 + t.rows;
            const int node0 = t.g * p.group_nodes;
            const int in_group = min(p.group_nodes, p.T - node0);
            const int ncols = (in_group + 31) & ~31;
            const uint32_t base = tmem + lane_addr + (uint32_t)acc * 256u;
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

// ---------------------------------------------------------------------------
// CTA-pair form: a cluster of two CTAs on two SMs runs 2-SM MMAs with M = 256
// vocabulary rows (128 per CTA) and N = up to 256 nodes.  Each CTA copies its
// own 128 W rows and HALF of the node group's H rows (the MMA reads the other
// half from the peer), so a K-chunk stage is at most 32 KB and six fit, and
// every SM streams half as much H per flop as the single-CTA form.
//   warp 0 (both)      producer; its copies complete on the FIRST CTA's full
//                      barriers, whose expected byte count covers both CTAs
//   warp 1 (first)     MMA issuer; its commits arrive on both CTAs' barriers
//   warps 2..5 (both)  epilogue on the CTA's own TMEM rows; the second CTA's
//                      warps release an accumulator on the first CTA's barrier
// Both CTAs always reach the two cluster barriers (after set-up and before
// exit); every other wait is bounded.
// ---------------------------------------------------------------------------
constexpr int kPairRows = 2 * kTileM;

struct LmPairItem {
    int row0, rows, g;     // the pair's rows [row0, row0 + rows), node group
};

// Items of a pair.  One node group: a contiguous, balanced vocabulary range
// (W is read once).  Several: items (tile, group), group fastest, dealt out
// round-robin -- pair p takes items p, p + npairs, ... -- so at any moment
// neighbouring pairs work on the same W tile for different node groups and
// each tile comes from HBM once and from L2 for the other groups.
struct LmPairWork {
    int r0, r1, pair, npairs, items;
    __device__ LmPairWork(const LmParams &p, int pair_, int npairs_) : pair(pair_), npairs(npairs_) {
        if (p.ngroups == 1) {
            r0 = (int)((long long)p.V * pair / npairs);
            r1 = (int)((long long)p.V * (pair + 1) / npairs);
            items = (r1 - r0 + kPairRows - 1) / kPairRows;
        } else {
            const long long total = (long long)((p.V + kPairRows - 1) / kPairRows) * p.ngroups;
            r0 = r1 = 0;
            items = (int)((total - pair + npairs - 1) / npairs);
        }
    }
    __device__ LmPairItem item(const LmParams &p, int k) const {
        LmPairItem t;
        if (p.ngroups == 1) {
            t.row0 = r0 + k * kPairRows;
            t.rows = min(kPairRows, r1 - t.row0);
            t.g = 0;
        } else {
            const long long i = pair + (long long)k * npairs;
            const int vt = (int)(i / p.ngroups);
            t.row0 = vt * kPairRows;
            t.rows = min(kPairRows, p.V - t.row0);
            t.g = (int)(i - (long long)vt * p.ngroups);
        }
        return t;
    }
};

__device__ __forceinline__ int pair_rows(const LmPairItem &t, int rank) {
    return max(0, min(kTileM, t.rows - rank * kTileM));
}
__device__ __forceinline__ uint32_t w_bytes(int rows) {
    return rows == kTileM ? kStageA : (uint32_t)((rows + kBoxRowsW - 1) / kBoxRowsW) * (kBoxRowsW * 128);
}

__global__ void __launch_bounds__(kLmThreads, 1)
lmhead_argmax_pair_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmW16,
                          const __grid_constant__ CUtensorMap tmH, const LmParams p) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int ep_fail;
    __shared__ unsigned long long red[kEpiWarps][kMaxGroupNodes];

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank();
    const LmPairWork work(p, blockIdx.x >> 1, gridDim.x >> 1);
    const int items = work.items;
    const int half_nodes = p.group_nodes / 2;         // H rows this CTA copies per item

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accf_bar[a], 1);
            mbar_init(&acce_bar[a], 2 * kEpiWarps);   // epilogue warps of both CTAs
        }
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        ep_fail = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_base_sh, 512);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmW);
        prefetch_tensormap(&tmW16);
        prefetch_tensormap(&tmH);
    }
    tc_fence_before();
    cluster_sync();          // both CTAs' barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_w = p.ngroups == 1 ? policy_evict_first() : policy_evict_normal();
            const uint64_t pol_h = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int it = 0; it < items && !abort_sh; ++it) {
                const LmPairItem t = work.item(p, it);
                const int my_rows = pair_rows(t, rank);
                const int my_row0 = t.row0 + rank * kTileM;
                const int in_group = min(p.group_nodes, p.T - t.g * p.group_nodes);
                const int nmma = (in_group + 15) & ~15;
                const int node0 = t.g * p.group_nodes + rank * (nmma / 2);
                // bytes both CTAs copy for one K-chunk (the first CTA expects them all)
                const uint32_t tx = 2u * (uint32_t)half_nodes * 128 + w_bytes(pair_rows(t, 0)) +
                                    (pair_rows(t, 1) > 0 ? w_bytes(pair_rows(t, 1)) : 0u);
                bool ok = true;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh)) {
                        set_abort(&abort_sh, p.status);
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + (size_t)stage * p.stage_bytes;
                    uint8_t *sb = sa + kStageA;
                    const uint32_t fbar = cluster_addr(&full_bar[stage], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], tx);
                    if (my_rows == kTileM) {
                        tma_load_2d_pair(sa, &tmW, fbar, kc * kKChunk, my_row0, pol_w);
                    } else {
                        for (int bx = 0; bx * kBoxRowsW < my_rows; ++bx)
                            tma_load_2d_pair(sa + bx * (kBoxRowsW * 128), &tmW16, fbar, kc * kKChunk,
                                             my_row0 + bx * kBoxRowsW, pol_w);
                    }
                    tma_load_2d_pair(sb, &tmH, fbar, kc * kKChunk, node0, pol_h);
                    ++issued;
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
            }
            if (abort_sh && rank == 0) {
                // let every load still in flight (both CTAs') land before exit
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
        // The whole warp runs the issue loop with warp-uniform operands (one
        // elected lane issues); lane 0 waits on the barriers and broadcasts.
        if (rank == 0) {
            auto wait1 = [&](uint64_t *bar, uint32_t parity) -> bool {
                int w = 1;
                if (lane == 0) w = mbar_wait(bar, parity, &abort_sh) ? 1 : 0;
                return __shfl_sync(0xffffffffu, w, 0) != 0;
            };
            const uint64_t da0 = desc_kmajor_sw128(smem_addr(smem));
            const uint64_t db0 = desc_kmajor_sw128(smem_addr(smem + kStageA));
            int stage = 0;
            uint32_t phase = 0;
            for (int it = 0; it < items; ++it) {
                const int acc = it & 1;
                const uint32_t use = (uint32_t)(it >> 1);
                if (!wait1(&acce_bar[acc], (use & 1) ^ 1)) {
                    if (lane == 0) set_abort(&abort_sh, p.status);
                    break;
                }
                tc_fence_after();
                const LmPairItem t = work.item(p, it);
                const int in_group = min(p.group_nodes, p.T - t.g * p.group_nodes);
                const uint32_t idn = idesc_bf16_f32(kPairRows, (in_group + 15) & ~15, false, false);
                const uint32_t d0 = tmem + (uint32_t)acc * 256u;
                bool ok = true;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!wait1(&full_bar[stage], phase)) {
                        if (lane == 0) set_abort(&abort_sh, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t soff = (uint64_t)((stage * p.stage_bytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < kKChunk / 16; ++kk)
                        mma_bf16_ss_pair_warp(d0, da0 + soff + (uint64_t)(kk * 2), db0 + soff + (uint64_t)(kk * 2),
                                              idn, (kc | kk) != 0);
                    mma_commit_pair_warp(&empty_bar[stage], 0x3);
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit_pair_warp(&accf_bar[acc], 0x3);
            }
            // every MMA issued above has finished before either CTA frees TMEM
            mma_commit_pair_warp(&drain_bar, 0x3);
        }
        if (lane == 0) {
            int zero = 0;
            mbar_wait(&drain_bar, 0, (volatile int *)&zero);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - 2;                     // 0..3
        const int sub = warp & 3;                    // TMEM lanes this warp may access
        const uint32_t lane_addr = (uint32_t)(sub * 32) << 16;
        const int et = threadIdx.x - 64;             // 0..127
        for (int it = 0; it < items; ++it) {
            const int acc = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            if (!mbar_wait(&accf_bar[acc], use & 1, &abort_sh)) {
                set_abort(&abort_sh, p.status);
                ep_fail = 1;
            }
            named_barrier(1, 32 * kEpiWarps);
            if (ep_fail) break;
            tc_fence_after();
            const LmPairItem t = work.item(p, it);
            const int my_rows = pair_rows(t, rank);
            const int v0 = t.row0 + rank * kTileM;
            const int v = v0 + sub * 32 + lane;
            const bool vvalid = v < v0 + my_rows;
            const int node0 = t.g * p.group_nodes;
            const int in_group = min(p.group_nodes, p.T - node0);
            const int ncols = (in_group + 31) & ~31;
            const uint32_t base = tmem + lane_addr + (uint32_t)acc * 256u;
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
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&acce_bar[acc]);
                else mbar_arrive_cluster(cluster_addr(&acce_bar[acc], 0));
            }
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

    __syncwarp();
    tc_fence_before();
    __threadfence();
    cluster_sync();          // both CTAs done with the pair's TMEM and shared memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
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

// Pairs of CTAs that can be resident at once for a given dynamic shared memory
// size (0 if clusters cannot be used).
static int pair_clusters(size_t smem) {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < 64 && cache[dev]) return cache[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 256);
    cfg.blockDim = dim3(kLmThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, lmhead_argmax_pair_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    if (dev < 64) cache[dev] = n > 0 ? n : -1;
    return n > 0 ? n : 0;
}

cudaError_t launch_lmhead_argmax(const uint16_t *hidden, const uint16_t *w, int T, int d, int V,
                                 int32_t *argmax, float *max_logit, void *ws, cudaStream_t st) {
    int32_t *status = nullptr;
    auto *keys = static_cast<unsigned long long *>(ws);
    LmParams p;
    p.T = T; p.d = d; p.V = V;
    p.kchunks = d / kKChunk;
    p.group_nodes = min(kMaxGroupNodes, (T + 15) & ~15);
    p.ngroups = (T + p.group_nodes - 1) / p.group_nodes;
    p.keys = keys;
    p.done = reinterpret_cast<unsigned int *>(keys + T);
    p.argmax = argmax;
    p.max_logit = max_logit;
    p.status = status;

    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(lmhead_argmax_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemBudget + 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(lmhead_argmax_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemBudget + 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;

    // CTA pairs: each CTA stages its 128 W rows and half of the group's H rows
    const uint32_t pair_stage = kStageA + (uint32_t)(p.group_nodes / 2) * 128;
    int pair_stages = kSmemBudget / (int)pair_stage;
    if (pair_stages > kMaxStages) pair_stages = kMaxStages;
    const size_t pair_smem = (size_t)pair_stages * pair_stage + 1024;
    // Up to 128 nodes the W stream from HBM bounds the kernel and single CTAs
    // stream it slightly better; above, the tensor pipe does and pairs feed it
    // with half the H traffic per SM and deeper stage rings.
    const int clusters = p.group_nodes > 128 ? pair_clusters(pair_smem) : 0;
    const bool use_pair = clusters > 0;

    CUtensorMap tmW, tmW16, tmH;
    if (!encode_tensor_map_2d(&tmW, w, (uint64_t)d, (uint64_t)V, (uint64_t)d * 2, kKChunk, kTileM))
        return cudaErrorInvalidValue;
    if (!encode_tensor_map_2d(&tmW16, w, (uint64_t)d, (uint64_t)V, (uint64_t)d * 2, kKChunk, kBoxRowsW))
        return cudaErrorInvalidValue;
    const int h_box = use_pair ? p.group_nodes / 2 : p.group_nodes;
    if (!encode_tensor_map_2d(&tmH, hidden, (uint64_t)d, (uint64_t)T, (uint64_t)d * 2, kKChunk, h_box))
        return cudaErrorInvalidValue;

    cudaError_t e = cudaMemsetAsync(keys, 0, lmhead_workspace_bytes(T, d, V), st);
    if (e != cudaSuccess) return e;
    if (use_pair) {
        p.stage_bytes = pair_stage;
        p.stages = pair_stages;
        const long long items = (long long)((V + kPairRows - 1) / kPairRows) * p.ngroups;
        long long pairs = clusters < sms / 2 ? clusters : sms / 2;
        if (pairs > items) pairs = items;
        e = launch_pdl_cluster(lmhead_argmax_pair_kernel, dim3((unsigned)(2 * pairs)), dim3(kLmThreads), pair_smem,
                               st, 2, tmW, tmW16, tmH, p);
    } else {
        p.stage_bytes = kStageA + (uint32_t)p.group_nodes * 128;
        p.stages = kSmemBudget / (int)p.stage_bytes;
        if (p.stages > kMaxStages) p.stages = kMaxStages;
        const size_t smem = (size_t)p.stages * p.stage_bytes + 1024;
        const long long items = (long long)((V + kTileM - 1) / kTileM) * p.ngroups;
        int grid = sms;
        if (grid > items) grid = (int)items;
        e = launch_pdl(lmhead_argmax_tc_kernel, dim3(grid), dim3(kLmThreads), smem, st, tmW, tmW16, tmH, p);
    }
    count_launches(1);
    return e;
}

}  // namespace jsv
