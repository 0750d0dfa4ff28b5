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
// An item is one vocabulary unit (up to 128 rows) x one group of up to 256
// nodes.  One CTA per SM at a time, 6 warps:
//   warp 0      TMA producer: the unit's W rows (one box) + the group's H
//               rows per 64-wide K chunk into a ring of shared-memory stages;
//               also asks cluster launch control for the next item
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, per-column argmax
//               across the unit's vocabulary rows (a transposing butterfly
//               of 64-bit keys), kept per node in shared memory
// Two accumulators alternate in TMEM, so the epilogue of one item overlaps
// the main loop of the next.
// Work split: the grid has one CTA per item; a running CTA that finishes an
// item cancels a CTA that has not started and takes its item (cluster launch
// control), so the items spread over whatever SMs are free -- the kernel
// starts beside the attention kernels of the step and takes their SMs as
// they finish.  Units are whole 16-row boxes, balanced so that with every SM
// free each CTA gets the same number of rows.  With one node group (up to
// 256 nodes) W, the dominant byte stream, is read exactly once; with several
// the items are ordered group fastest, so CTAs working at the same time
// share a W unit through L2.
//
// Node groups above 128 (tensor-bound) run on CTA pairs with 2-SM MMAs; see
// the pair kernel below.
//
// Cross-CTA reduction: a 64-bit key per node whose high word is the fp32
// value mapped to an order-preserving unsigned integer and whose low word is
// ~index; atomicMax keeps the largest value and, among equal values, the
// smallest index.  Each CTA merges its per-node maxima into the keys once,
// after waiting for the previous launch on the stream (the main loop reads
// only W and H, so it does not wait).  The CTA that completes the count of
// finished work (a counter in the workspace) writes every node's argmax and
// maximum and zeroes the keys and the counter for the next call.
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
    int units;         // single-CTA form: vocabulary units (see lm_unit)
    int unit_b;        // 16-row boxes of a short unit
    int unit_rem;      // units [0, unit_rem) take unit_b + 1 boxes
    int tiles;         // single-CTA form: 128-row W tiles a unit may span (1 or 2)
    unsigned long long *keys;
    unsigned int *done;        // work finished so far (zero between calls)
    int32_t *argmax;
    float *max_logit;
    int32_t *status;           // device status word or NULL (JSV_ERR_TIMEOUT on a wait that gave up)
    uint64_t inject_ns;        // failure-detection self-test: 0, or the limit of an injected wait
};

// Single-CTA form: the vocabulary is cut into `units` runs of whole 16-row
// boxes, unit_b or unit_b + 1 boxes each, at most 8 per 128-row MMA tile and
// `tiles` tiles per unit, with the unit count a multiple of the SM count
// where the vocabulary allows; the last run may reach past V, where the
// tensor map fills zeros and the epilogue ignores the rows.  An item is one
// unit x one node group (group fastest); the grid has one CTA per item.
//
// Two tiles per unit: every K-chunk stage holds both tiles' W rows and ONE
// copy of the group's H rows, and each K-step issues one MMA per tile into
// its own TMEM accumulator.  The cost of a unit is set mostly by its K-chunk
// stages (each brings the group's H rows from L2 and takes a full barrier
// round trip), not by its W rows, so a unit twice as tall halves that cost
// per vocabulary row.
struct LmUnit {
    int row0, boxes;
};

// W tensor maps with box heights of 1..8 16-row boxes (one per height).
struct LmWMaps {
    CUtensorMap m[kTileM / kBoxRowsW];
};

__device__ __forceinline__ LmUnit lm_unit(const LmParams &p, int u) {
    LmUnit t;
    const int big = p.unit_b + 1;
    if (u < p.unit_rem) {
        t.row0 = u * big * kBoxRowsW;
        t.boxes = big;
    } else {
        t.row0 = (p.unit_rem * big + (u - p.unit_rem) * p.unit_b) * kBoxRowsW;
        t.boxes = p.unit_b;
    }
    return t;
}

__device__ __forceinline__ void set_abort(volatile int *abort, int32_t *status) {
    *abort = 1;
    if (status) atomicCAS(status, 0, JSV_ERR_TIMEOUT);
}

// The same in a CTA pair: the peer's flag is raised too (distributed shared
// memory; both CTAs are alive until their last cluster barrier), so that both
// stop issuing work instead of running into their own wait limits.
__device__ __forceinline__ void set_abort_pair(volatile int *abort, int32_t *status) {
    set_abort(abort, status);
    st_shared_cluster_u32((const void *)abort, cluster_ctarank() ^ 1u, 1u);
}

// Failure-detection self-test (jsv_selftest_lmhead_timeout): the producer of
// the first CTA (or CTA pair) waits, before it issues any copy, on a barrier
// nothing signals, with the injected limit.  It gives up, reports the timeout
// and unwinds like any timed-out wait; nothing of its own is in flight then.
__device__ __forceinline__ bool injected_wait_gave_up(const LmParams &p, uint64_t *bar, volatile int *abort,
                                                     unsigned first_ctas) {
    if (p.inject_ns == 0 || blockIdx.x >= first_ctas) return false;
    return !mbar_wait(bar, 0, abort, p.inject_ns);
}

// Answers of cluster launch control: the CTA's k-th item is blockIdx.x for
// k = 0; the answer carrying item k + 1 lands in slot k % kClcSlots, in
// phase (k / kClcSlots) & 1.  Every role reads every answer.
constexpr int kClcSlots = 4;
constexpr int kClcReaders = 2 + kEpiWarps;     // producer, MMA issuer, epilogue warps

// Dynamic scheduling: a running CTA that finishes an item cancels a CTA of
// the grid that has not started yet and takes its item instead, so CTAs
// that start late (their SM was still held by an earlier kernel) end up
// with fewer items and all finish together.  Completion is counted in items:
// each CTA adds the items it took, and the CTA that brings the count to the
// grid size reduces the keys.
__global__ void __launch_bounds__(kLmThreads, 1)
lmhead_argmax_tc_kernel(const __grid_constant__ LmWMaps tmW, const __grid_constant__ CUtensorMap tmH,
                        const LmParams p) {
    pdl_allow_dependents();
    // With one node group, nothing before the final reduction touches memory
    // that an earlier launch on the stream may still be using (W and hidden
    // are only read; keys live in shared memory until then), so the wait for
    // that launch moves to the reduction and the main loop overlaps it.
    const bool late_wait = p.ngroups == 1;
    if (!late_wait) pdl_wait_predecessor();
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
    __shared__ __align__(8) uint64_t accf_bar[2], acce_bar[2], drain_bar;
    __shared__ __align__(8) uint64_t clc_full[kClcSlots], clc_empty[kClcSlots], inject_bar;
    __shared__ __align__(16) uint4 clc_resp[kClcSlots];
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int ep_fail;
    __shared__ int claimed_sh;
    __shared__ unsigned long long red[kEpiWarps][kMaxGroupNodes];
    __shared__ unsigned long long best[kMaxGroupNodes];     // this CTA's best key per node (one group)

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accf_bar[a], 1);
            mbar_init(&acce_bar[a], kEpiWarps);
        }
        for (int s = 0; s < kClcSlots; ++s) {
            mbar_init(&clc_full[s], 1);
            mbar_init(&clc_empty[s], kClcReaders);
        }
        mbar_init(&drain_bar, 1);
        mbar_init(&inject_bar, 1);
        abort_sh = 0;
        ep_fail = 0;
        claimed_sh = 1;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < kTileM / kBoxRowsW; ++i) prefetch_tensormap(&tmW.m[i]);
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
            int item = blockIdx.x, claimed = 1;
            int pend_slot = -1;                  // an answer still on its way
            uint32_t pend_phase = 0;
            if (injected_wait_gave_up(p, &inject_bar, &abort_sh, 1)) set_abort(&abort_sh, p.status);
            for (int k = 0; !abort_sh; ++k) {
                const int cs = k % kClcSlots;
                const uint32_t cph = (uint32_t)(k / kClcSlots) & 1u;
                // ask for the next item while this one streams in
                if (!mbar_wait(&clc_empty[cs], cph ^ 1, &abort_sh)) {
                    set_abort(&abort_sh, p.status);
                    break;
                }
                mbar_arrive_expect_tx(&clc_full[cs], 16);
                clc_try_cancel(&clc_resp[cs], &clc_full[cs]);
                pend_slot = cs;
                pend_phase = cph;
                const LmUnit t = lm_unit(p, item / p.ngroups);
                const int node0 = (item % p.ngroups) * p.group_nodes;
                const int boxes0 = min(t.boxes, kTileM / kBoxRowsW), boxes1 = t.boxes - boxes0;
                const uint32_t tx = (uint32_t)p.group_nodes * 128 + (uint32_t)t.boxes * (kBoxRowsW * 128);
                bool ok = true;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh)) {
                        set_abort(&abort_sh, p.status);
                        ok = false;
                        break;
                    }
                    uint8_t *sa = smem + (size_t)stage * p.stage_bytes;
                    mbar_arrive_expect_tx(&full_bar[stage], tx);
                    tma_load_2d_hint(sa, &tmW.m[boxes0 - 1], &full_bar[stage], kc * kKChunk, t.row0, pol_w);
                    if (boxes1 > 0)
                        tma_load_2d_hint(sa + kStageA, &tmW.m[boxes1 - 1], &full_bar[stage], kc * kKChunk,
                                         t.row0 + kTileM, pol_w);
                    tma_load_2d_hint(sa + p.tiles * kStageA, &tmH, &full_bar[stage], kc * kKChunk, node0, pol_h);
                    ++issued;
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                if (!mbar_wait(&clc_full[cs], cph, &abort_sh)) {
                    set_abort(&abort_sh, p.status);
                    break;
                }
                pend_slot = -1;
                int next = 0;
                const bool got = clc_query(&clc_resp[cs], next);
                fence_async_smem();
                mbar_arrive(&clc_empty[cs]);
                if (!got) break;
                item = next;
                ++claimed;
            }
            int zero = 0;
            if (pend_slot >= 0) {
                // an answer is still on its way: it must land before the CTA
                // exits, and an item it carries counts as taken (unprocessed
                // after an abort, but the completion count still closes)
                if (mbar_wait(&clc_full[pend_slot], pend_phase, (volatile int *)&zero)) {
                    int next = 0;
                    if (clc_query(&clc_resp[pend_slot], next)) ++claimed;
                }
            }
            if (abort_sh) {
                // let every load still in flight land before the CTA exits
                const long long back = issued < p.stages ? issued : p.stages;
                int s = stage;
                uint32_t ph = phase;
                for (long long i = 0; i < back; ++i) {
                    if (s == 0) { s = p.stages; ph ^= 1; }
                    --s;
                    mbar_wait(&full_bar[s], ph, (volatile int *)&zero);
                }
            }
            claimed_sh = claimed;
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int item = blockIdx.x;
            for (int k = 0; !abort_sh; ++k) {
                const int acc = k & 1;
                const uint32_t use = (uint32_t)(k >> 1);
                if (!mbar_wait(&acce_bar[acc], (use & 1) ^ 1, &abort_sh)) {
                    set_abort(&abort_sh, p.status);
                    break;
                }
                tc_fence_after();
                const int node0 = (item % p.ngroups) * p.group_nodes;
                const int in_group = min(p.group_nodes, p.T - node0);
                const uint32_t idn = idesc_bf16_f32(kTileM, (in_group + 15) & ~15, false, false);
                const uint32_t d0 = tmem + (uint32_t)acc * 256u;
                // a unit's second tile (rows 128..) accumulates 128 columns on
                const bool two = lm_unit(p, item / p.ngroups).boxes > kTileM / kBoxRowsW;
                bool ok = true;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&full_bar[stage], phase, &abort_sh)) {
                        set_abort(&abort_sh, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + (size_t)stage * p.stage_bytes);
                    const uint32_t sb = sa + (uint32_t)p.tiles * kStageA;
#pragma unroll
                    for (int kk = 0; kk < kKChunk / 16; ++kk) {
                        const uint64_t db = desc_kmajor_sw128(sb + kk * 32);
                        mma_bf16_ss(d0, desc_kmajor_sw128(sa + kk * 32), db, idn, (kc | kk) != 0);
                        if (two)
                            mma_bf16_ss(d0 + (uint32_t)kTileM, desc_kmajor_sw128(sa + kStageA + kk * 32), db, idn,
                                        (kc | kk) != 0);
                    }
                    mma_commit(&empty_bar[stage]);
                    if (++stage == p.stages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(&accf_bar[acc]);
                const int cs = k % kClcSlots;
                if (!mbar_wait(&clc_full[cs], (uint32_t)(k / kClcSlots) & 1u, &abort_sh)) {
                    set_abort(&abort_sh, p.status);
                    break;
                }
                int next = 0;
                const bool got = clc_query(&clc_resp[cs], next);
                fence_async_smem();
                mbar_arrive(&clc_empty[cs]);
                if (!got) break;
                item = next;
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
        for (int c = et; c < kMaxGroupNodes; c += 32 * kEpiWarps) best[c] = 0ull;
        int item = blockIdx.x;
        for (int k = 0;; ++k) {
            const int acc = k & 1;
            const uint32_t use = (uint32_t)(k >> 1);
            if (!mbar_wait(&accf_bar[acc], use & 1, &abort_sh)) {
                set_abort(&abort_sh, p.status);
                ep_fail = 1;
            }
            named_barrier(1, 32 * kEpiWarps);
            if (ep_fail) break;
            tc_fence_after();
            const LmUnit t = lm_unit(p, item / p.ngroups);
            const int row_end = min(t.row0 + t.boxes * kBoxRowsW, p.V);
            const int ntiles = t.boxes > kTileM / kBoxRowsW ? 2 : 1;
            const int node0 = (item % p.ngroups) * p.group_nodes;
            const int in_group = min(p.group_nodes, p.T - node0);
            const int ncols = (in_group + 31) & ~31;
            for (int tile = 0; tile < ntiles; ++tile) {
                const int v = t.row0 + tile * kTileM + sub * 32 + lane;
                const bool vvalid = v < row_end;
                const uint32_t base = tmem + lane_addr + (uint32_t)acc * 256u + (uint32_t)(tile * kTileM);
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
                    red[ew][c0 + lane] = tile == 0 ? x[0] : umax64(red[ew][c0 + lane], x[0]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce_bar[acc]);
            named_barrier(1, 32 * kEpiWarps);
            for (int c = et; c < in_group; c += 32 * kEpiWarps) {
                unsigned long long key = red[0][c];
#pragma unroll
                for (int w = 1; w < kEpiWarps; ++w) key = umax64(key, red[w][c]);
                if (late_wait)
                    best[c] = umax64(best[c], key);
                else if (key)
                    atomicMax(&p.keys[node0 + c], key);
            }
            // the next item (every epilogue warp reads the same answer)
            const int cs = k % kClcSlots;
            int next = 0;
            bool got = false;
            if (mbar_wait(&clc_full[cs], (uint32_t)(k / kClcSlots) & 1u, &abort_sh)) {
                got = clc_query(&clc_resp[cs], next);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&clc_empty[cs]);
            } else {
                set_abort(&abort_sh, p.status);
                ep_fail = 1;
            }
            named_barrier(1, 32 * kEpiWarps);
            if (ep_fail || !got) break;
            item = next;
        }
        if (late_wait) {
            // the previous launch on the stream has completed: the keys are
            // free (and zero), so this CTA's maxima go out now
            pdl_wait_predecessor();
            for (int c = et; c < p.T; c += 32 * kEpiWarps)
                if (best[c]) atomicMax(&p.keys[c], best[c]);
        }
    }

    tc_fence_before();
    __threadfence();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    // The CTA that completes the item count turns every node's key into its
    // argmax and leaves the workspace zeroed for the next call.
    __shared__ int is_last;
    if (threadIdx.x == 0) {
        const unsigned total = (unsigned)p.units * (unsigned)p.ngroups;
        is_last = atomicAdd(p.done, (unsigned)claimed_sh) + (unsigned)claimed_sh == total;
    }
    __syncthreads();
    if (is_last) {
        pdl_wait_predecessor();
        __threadfence();
        for (int t = threadIdx.x; t < p.T; t += blockDim.x) {
            const unsigned long long key = atomicExch(&p.keys[t], 0ull);
            p.argmax[t] = (int32_t)(~(uint32_t)(key & 0xffffffffull));
            if (p.max_logit) p.max_logit[t] = key_value(key);
        }
        if (threadIdx.x == 0) atomicExch(p.done, 0u);
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
    int row0, rows;        // the pair's vocabulary rows [row0, row0 + rows)
    int node0, nodes;      // its nodes [node0, node0 + nodes)
};

// Items of a pair.  An item is one 256-row vocabulary unit x one node group
// (group fastest): with several groups, consecutive items share a W unit, so
// at any moment neighbouring pairs read the same unit and it comes from HBM
// once and from L2 for the other groups; with one group W is read once.
// The `base` = items / npairs whole rounds are dealt round-robin (pair p takes
// items p, p + npairs, ...).  The `rem` items left over would leave most pairs
// idle for a last round -- a 2-SM MMA costs M = 256 rows and N = the group's
// nodes whatever the rows it holds -- so they are cut by nodes into pieces of
// piece_nodes nodes (16-node blocks, sized so that there are about as many
// pieces as pairs), also dealt round-robin.  A piece's pair still copies a
// full H box per CTA (rows past T read as zeros); its MMA reads the first
// piece_nodes / 2 rows of each.
struct LmPairWork {
    int pair, npairs, items;
    int base, rem, piece_nodes, pieces;
    __device__ __forceinline__ void item_geometry(const LmParams &p, int i, int &row0, int &node0, int &nodes) const {
        const int vt = i / p.ngroups, g = i - vt * p.ngroups;
        row0 = vt * kPairRows;
        node0 = g * p.group_nodes;
        nodes = min(p.group_nodes, p.T - node0);
    }
    __device__ LmPairWork(const LmParams &p, int pair_, int npairs_) : pair(pair_), npairs(npairs_) {
        const int total = ((p.V + kPairRows - 1) / kPairRows) * p.ngroups;
        base = total / npairs;
        rem = total - base * npairs;
        const int group_blocks = (p.group_nodes + 15) / 16;
        piece_nodes = 16 * max(1, (group_blocks * rem + npairs - 1) / npairs);
        pieces = 0;
        for (int r = 0; r < rem; ++r) {
            int row0, node0, nodes;
            item_geometry(p, base * npairs + r, row0, node0, nodes);
            pieces += (nodes + piece_nodes - 1) / piece_nodes;
        }
        items = base + (pair < pieces ? (pieces - pair + npairs - 1) / npairs : 0);
    }
    __device__ LmPairItem item(const LmParams &p, int k) const {
        LmPairItem t;
        if (k < base) {
            item_geometry(p, pair + k * npairs, t.row0, t.node0, t.nodes);
        } else {
            // piece q: find its leftover item by walking the items' piece counts
            int q = pair + (k - base) * npairs;
            int r = 0, row0 = 0, node0 = 0, nodes = 0;
            for (; r < rem; ++r) {
                item_geometry(p, base * npairs + r, row0, node0, nodes);
                const int nb = (nodes + piece_nodes - 1) / piece_nodes;
                if (q < nb) break;
                q -= nb;
            }
            t.row0 = row0;
            t.node0 = node0 + q * piece_nodes;
            t.nodes = min(piece_nodes, nodes - q * piece_nodes);
        }
        t.rows = min(kPairRows, p.V - t.row0);
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
    __shared__ __align__(8) uint64_t inject_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int ep_fail;
    __shared__ int issued_sh;                         // K-chunk stages this CTA's producer issued
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
        mbar_init(&inject_bar, 1);
        abort_sh = 0;
        ep_fail = 0;
        issued_sh = 0;
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
            int issued = 0;
            if (injected_wait_gave_up(p, &inject_bar, &abort_sh, 2)) set_abort_pair(&abort_sh, p.status);
            for (int it = 0; it < items && !abort_sh; ++it) {
                const LmPairItem t = work.item(p, it);
                const int my_rows = pair_rows(t, rank);
                const int my_row0 = t.row0 + rank * kTileM;
                const int nmma = (t.nodes + 15) & ~15;
                const int node0 = t.node0 + rank * (nmma / 2);
                // bytes both CTAs copy for one K-chunk (the first CTA expects them all)
                const uint32_t tx = 2u * (uint32_t)half_nodes * 128 + w_bytes(pair_rows(t, 0)) +
                                    (pair_rows(t, 1) > 0 ? w_bytes(pair_rows(t, 1)) : 0u);
                bool ok = true;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_sh)) {
                        set_abort_pair(&abort_sh, p.status);
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
            issued_sh = issued;
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
                    if (lane == 0) set_abort_pair(&abort_sh, p.status);
                    break;
                }
                tc_fence_after();
                const LmPairItem t = work.item(p, it);
                const uint32_t idn = idesc_bf16_f32(kPairRows, (t.nodes + 15) & ~15, false, false);
                const uint32_t d0 = tmem + (uint32_t)acc * 256u;
                bool ok = true;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!wait1(&full_bar[stage], phase)) {
                        if (lane == 0) set_abort_pair(&abort_sh, p.status);
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
                set_abort_pair(&abort_sh, p.status);
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
            const int node0 = t.node0;
            const int in_group = t.nodes;
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
    cluster_sync();          // both CTAs done with the pair's TMEM; producers' issue counts published
    // After an abort, copies may still be in flight into either CTA's shared
    // memory.  Every copy of a stage completes on the first CTA's barrier, so
    // its producer waits for each stage either CTA issued (the last `stages`
    // of them), first completing by hand the bytes of a CTA that never issued
    // its part of that stage and arming a stage only the second CTA issued.
    // Both CTAs then meet again, so neither exits with its copies in flight.
    const bool any_abort = abort_sh || ld_shared_cluster_u32((const void *)&abort_sh, (uint32_t)rank ^ 1u);
    if (any_abort) {
        if (rank == 0 && warp == 0 && lane == 0) {
            const int n0 = issued_sh, n1 = (int)ld_shared_cluster_u32(&issued_sh, 1);
            const int n = n0 > n1 ? n0 : n1;
            int zero = 0;
            for (int i = n - p.stages > 0 ? n - p.stages : 0; i < n; ++i) {
                const int s = i % p.stages;
                const uint32_t ph = (uint32_t)((i / p.stages) & 1);
                const LmPairItem t = work.item(p, i / p.kchunks);
                const uint32_t b0 = (uint32_t)half_nodes * 128 + w_bytes(pair_rows(t, 0));
                const uint32_t b1 = (uint32_t)half_nodes * 128 + (pair_rows(t, 1) > 0 ? w_bytes(pair_rows(t, 1)) : 0u);
                if (i >= n0) mbar_arrive_expect_tx(&full_bar[s], b1);      // armed by neither: rank 1's part only
                else if (i >= n1) mbar_complete_tx(&full_bar[s], b1);      // rank 1's part never issued
                mbar_wait(&full_bar[s], ph, (volatile int *)&zero);
            }
        }
        __syncwarp();
        cluster_sync();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, 512);
    }
    // the last CTA to finish turns every node's key into its argmax and
    // leaves the workspace zeroed for the next call
    __shared__ int is_last;
    if (threadIdx.x == 0) is_last = atomicAdd(p.done, 1u) == (unsigned)(gridDim.x - 1);
    __syncthreads();
    if (is_last) {
        __threadfence();
        for (int t = threadIdx.x; t < p.T; t += blockDim.x) {
            const unsigned long long k = atomicExch(&p.keys[t], 0ull);
            p.argmax[t] = (int32_t)(~(uint32_t)(k & 0xffffffffull));
            if (p.max_logit) p.max_logit[t] = key_value(k);
        }
        if (threadIdx.x == 0) atomicExch(p.done, 0u);
    }
}

size_t lmhead_workspace_bytes(int T, int d, int V) {
    (void)d; (void)V;
    return (size_t)T * sizeof(unsigned long long) + sizeof(unsigned long long);   // keys + done counter
}

// Pairs of CTAs that can be resident at once for a given dynamic shared memory
// size (0 if clusters cannot be used).
static int pair_clusters(size_t smem) {
    // several host threads may fill an entry at once; they store the same value
    static std::atomic<int> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
    if (dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c) return c > 0 ? c : 0;
    }
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
    if (dev < 64) cache[dev].store(n > 0 ? n : -1, std::memory_order_relaxed);
    return n > 0 ? n : 0;
}

cudaError_t launch_lmhead_argmax(const uint16_t *hidden, const uint16_t *w, int T, int d, int V,
                                 int32_t *argmax, float *max_logit, void *ws, int32_t *status,
                                 uint64_t inject_ns, cudaStream_t st) {
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
    p.inject_ns = inject_ns;

    static PerDeviceOnce attr_once;
    cudaError_t ae = attr_once.run([]() {
        cudaError_t e = cudaFuncSetAttribute(lmhead_argmax_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemBudget + 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(lmhead_argmax_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemBudget + 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(lmhead_argmax_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(lmhead_argmax_pair_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        return e;
    });
    if (ae != cudaSuccess) return ae;
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

    // The workspace arrives zeroed (first use) or as the previous call left
    // it (zeroed by that call's last CTA), so no clearing launch is needed.
    cudaError_t e = cudaSuccess;
    if (use_pair) {
        p.stage_bytes = pair_stage;
        p.stages = pair_stages;
        const long long items = (long long)((V + kPairRows - 1) / kPairRows) * p.ngroups;
        long long pairs = clusters < sms / 2 ? clusters : sms / 2;
        if (pairs > items) pairs = items;
        e = launch_pdl_cluster(lmhead_argmax_pair_kernel, dim3((unsigned)(2 * pairs)), dim3(kLmThreads), pair_smem,
                               st, 2, tmW, tmW16, tmH, p);
    } else {
        // two W tiles per unit when both accumulators of a buffer fit in its
        // 256 TMEM columns (up to 128 nodes)
        p.tiles = p.group_nodes <= kTileM ? 2 : 1;
        p.stage_bytes = (uint32_t)p.tiles * kStageA + (uint32_t)p.group_nodes * 128;
        p.stages = kSmemBudget / (int)p.stage_bytes;
        if (p.stages > kMaxStages) p.stages = kMaxStages;
        const size_t smem = (size_t)p.stages * p.stage_bytes + 1024;
        // vocabulary units of whole 16-row boxes, at most 8 per tile, as many
        // units per SM as that needs
        const long long max_boxes = (long long)p.tiles * (kTileM / kBoxRowsW);
        const long long boxes = ((long long)V + kBoxRowsW - 1) / kBoxRowsW;
        const long long per_sm = (boxes + max_boxes * sms - 1) / (max_boxes * sms);
        long long units = per_sm * sms;
        if (units > boxes) units = boxes;
        if (units * p.ngroups > 0x7fffffffLL) return cudaErrorInvalidValue;
        p.units = (int)units;
        p.unit_b = (int)(boxes / units);
        p.unit_rem = (int)(boxes - (long long)p.unit_b * units);
        LmWMaps maps;
        for (int i = 0; i < kTileM / kBoxRowsW; ++i)
            if (!encode_tensor_map_2d(&maps.m[i], w, (uint64_t)d, (uint64_t)V, (uint64_t)d * 2, kKChunk,
                                      (i + 1) * kBoxRowsW))
                return cudaErrorInvalidValue;
        e = launch_pdl(lmhead_argmax_tc_kernel, dim3((unsigned)(units * p.ngroups)), dim3(kLmThreads), smem, st,
                       maps, tmH, p);
    }
    count_launches(1);
    return e;
}

}  // namespace jsv
