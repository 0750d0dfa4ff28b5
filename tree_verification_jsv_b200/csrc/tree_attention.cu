// Tree-causal attention over a paged KV prefix on tcgen05 tensor cores.
//
// JetSpec README, "JetSpec / Overview": the whole draft tree is verified in
// one forward pass under a tree-causal mask.  Node i of request b attends to
// prefix slots [0, P) and to slot P + j for every ancestor-or-self j of i.
//
// Work decomposition (one CTA per unit):
//   (request b, KV head g, tile of 256 query rows, KV split s)
// Query rows of (b, g) pack the G = Hq/Hkv heads that share KV head g:
// row r <-> node r / G, head g*G + r % G, so every K/V tile loaded serves
// 256 query rows (GQA packing).  The 256 rows form two 128-row groups that
// take turns on the tensor core.  The prefix is cut into 128-key tiles that
// start on page boundaries, followed by the tree tiles, which cover slots
// [P & ~15, P + N) and apply the ancestor mask; split s takes a balanced
// contiguous run of these tiles (a split that holds tree tiles builds the
// ancestor bitsets).  A request takes as many splits as its tile count
// needs at about C tiles each (at most S, the largest request's count).
// Each split writes an unnormalised fp32 partial (O, row max, row sum); a
// small combine kernel merges the splits with log-sum-exp rescaling and
// rounds to bf16.  A request with one split writes its rows in bf16 from
// this kernel, and the combine skips it.  When every request has one split
// and the batch is small, the CTAs take the units longest first.
//
// Per CTA, 12 warps (three warpgroups):
//   warp 0      TMA producer: Q once, then K and V of each 128-key tile, one
//               16-slot page x 64-dim box per copy, into a 2-stage ring; the
//               warp looks up the next tile's pages while it waits for a stage
//   warp 1      TMEM allocator and single-thread MMA issuer, in the order
//               S0_0 S1_0 | PV0_0 S0_1 PV1_0 S1_1 | PV0_1 S0_2 ...
//               (Sg_j = Q_g K_j^T, PVg_j: O_g += P_g V_j with P read from TMEM)
//   warps 2, 3  idle (they complete the first warpgroup, which hands most of
//               its registers to the other two)
//   warps 4..7  softmax of row group 0, warps 8..11 of row group 1: one query
//               row per thread, the whole 128-column row of S read from TMEM
//               into registers at once; masked online softmax in the log2
//               domain (packed f32x2 arithmetic, three-input max); P_j (bf16)
//               is written over its own S buffer in TMEM;
//               O is rescaled in TMEM only when the running max grows by
//               more than 8 (2^8), which keeps exp2 arguments bounded
// While one group computes its softmax the tensor core runs the other
// group's products.  The overlap is partial: a group's softmax (about 1,950
// cycles a tile on B200) outlasts the other group's 16 MMAs (about 1,250), so
// a tile takes about 3,600 cycles against 2,048 of tensor work, bound by the
// cycle S -> softmax -> P -> PV, S of the next tile.
// TMEM columns: S/P of group 0 [0,128), of group 1 [128,256); O of group 0
// [256, 256+D), of group 1 [256+D, 256+2D).
// Shared memory: Q (2 groups x 16 KB per 64 dims), 2 x (K, V) stages.
#include "jsv_internal.cuh"
#include "sm100.cuh"

#include <math.h>
#include <type_traits>
#include <string.h>

namespace jsv {

using namespace sm100;

constexpr int kGroups = 2;
constexpr int kGroupRows = 128;
constexpr int kRowsPerCta = kGroups * kGroupRows;
constexpr int kSoftmaxWarp0 = 4;              // warps 0..3: producer, MMA, two idle
constexpr int kAttnThreads = 32 * kSoftmaxWarp0 + kGroups * 128;
// registers a thread after the split (launch: 168 for all 12 warps); the
// three warps of an SMSP hold 56 + 224 + 224 of its 512 registers a lane, and
// 128 x 56 + 256 x 224 equals the 384 x 168 the CTA is launched with
constexpr int kRegsControl = 56;
constexpr int kRegsSoftmax = 224;
constexpr int kKeyTile = 128;
constexpr int kStages = 2;
constexpr int kMaxTreeWords = 16;          // 512 nodes
constexpr float kRescaleThreshold = 8.0f;  // log2 units

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction per pair).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}


struct AttnParams {
    BatchArgs a;
    const uint16_t *q;
    uint16_t *out;         // [T][Hq][D] bf16, written here for rows that are not split
    float scale_log2;
    int S;                 // most splits of a request (grid dimension y)
    int C;                 // key tiles a split aims at
    int q_tma;             // 1: Q is copied by TMA (G divides 128), 0: by the softmax warps
    float *ws_o;           // [S][T*Hq][D]
    float *ws_ml;          // [S][T*Hq][2]
};

// Splits of a request with `total` key tiles: about C tiles each, at most S,
// so that short requests of a ragged batch take fewer CTAs than long ones.
__device__ __forceinline__ int request_splits(int total, int C, int S) {
    return max(1, min(S, (total + C - 1) / C));
}

// Key tiles of a request: prefix tiles, then tree tiles from the page
// boundary at or below P.
__device__ __forceinline__ int request_tiles(const Request &r) {
    return (r.P + kKeyTile - 1) / kKeyTile + (r.P + r.n - (r.P & ~15) + kKeyTile - 1) / kKeyTile;
}

// Longest-first order for batches of up to kLptMaxReqs requests (used when
// the batch's largest request takes one split).  The CTAs
// of a launch start in block order, so block L takes the L-th work unit
// (request, KV head, row tile, split) with the requests sorted by tiles per
// split, largest first (ties: lower request index first), and the blocks
// past the last unit return at once: long units start first, short ones fill
// the SMs as they free up, and no empty unit sits between them.  One warp
// computes it from the request geometry; (b, unit index within b) or b = -1.
constexpr int kLptMaxReqs = 64;

__device__ __forceinline__ void lpt_unit(const AttnParams &prm, int L, int lane, int *s_units, int *s_b,
                                         int &ub, int &uloc) {
    const BatchArgs &a = prm.a;
    const int G = a.Hq / a.Hkv;
    int work[2], units[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int rb = lane + 32 * k;
        work[k] = -1;
        units[k] = 0;
        Request q;
        if (rb < a.B && load_request(a, rb, q)) {
            const int K = request_tiles(q);
            const int sb = request_splits(K, prm.C, prm.S);
            units[k] = a.Hkv * ((q.n * G + kRowsPerCta - 1) / kRowsPerCta) * sb;
            work[k] = (K + sb - 1) / sb;
        }
    }
    int rank[2] = {0, 0};
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        for (int j = 0; j < 32; ++j) {
            const int wj = __shfl_sync(0xffffffffu, work[kk], j), bj = j + 32 * kk;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int bi = lane + 32 * k;
                if (bj < a.B && (wj > work[k] || (wj == work[k] && bj < bi))) ++rank[k];
            }
        }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        if (lane + 32 * k < a.B) {
            s_units[rank[k]] = units[k];
            s_b[rank[k]] = lane + 32 * k;
        }
    }
    __syncwarp();
    // exclusive prefix of the sorted units: lane l holds entries 2l, 2l + 1
    const int e0 = 2 * lane, e1 = 2 * lane + 1;
    const int u0 = e0 < a.B ? s_units[e0] : 0, u1 = e1 < a.B ? s_units[e1] : 0;
    int incl = u0 + u1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    const int excl = incl - u0 - u1;
    int fb = -1, fl = 0;
    if (L >= excl && L < excl + u0) {
        fb = s_b[e0];
        fl = L - excl;
    } else if (L >= excl + u0 && L < incl) {
        fb = s_b[e1];
        fl = L - excl - u0;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, fb >= 0);
    ub = hit ? __shfl_sync(0xffffffffu, fb, __ffs(hit) - 1) : -1;
    uloc = hit ? __shfl_sync(0xffffffffu, fl, __ffs(hit) - 1) : 0;
}

template <int D>
struct AttnSmem {
    static constexpr int kQGroupBytes = kGroupRows * D * 2;    // one row group's Q
    static constexpr int kQBytes = kGroups * kQGroupBytes;
    static constexpr int kKVBytes = kKeyTile * D * 2;          // one K (or V) tile
    static constexpr int kStageBytes = 2 * kKVBytes;
    static constexpr int kTotal = kQBytes + kStages * kStageBytes;
};

// Byte offset of 16-byte chunk `c` of row `r` in a K-major SW128 operand
// region (rows of 128 B, 8-row atoms; chunk index XOR row % 8).
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// The MMA issuer: one thread of the CTA issues every tcgen05.mma.  S of a
// group reuses the TMEM of that group's previous P; the PV that reads it was
// issued earlier and MMAs run in issue order.
//
// Instantiated per group count so that every TMEM address and descriptor
// offset is a compile-time constant added to a base formed once: this
// thread's instruction stream between two MMAs is on the tensor pipe's
// critical path (with the group index and the addresses computed at run time
// the MMAs issued about 1.3x slower).  A descriptor's start-address field
// holds (address >> 4) in 14 bits; shared memory ends below 256 KB, so adding
// an offset to a base descriptor never carries out of the field.
template <int D, int NG>
__device__ __forceinline__ void attention_mma_loop(uint32_t tmem, uint32_t aQ, uint32_t aKV, int ntiles,
                                                   uint64_t *k_full, uint64_t *v_full, uint64_t *k_empty,
                                                   uint64_t *v_empty, uint64_t *s_full, uint64_t *p_full,
                                                   uint64_t *o_done, uint64_t *q_ready, uint64_t *drain_bar,
                                                   volatile int *abort_sh, int32_t *dev_status) {
    using L = AttnSmem<D>;
    constexpr uint32_t id_s = idesc_bf16_f32(128, kKeyTile, false, false);
    constexpr uint32_t id_o = idesc_bf16_f32(128, D, false, true);
    constexpr uint32_t kStageStep = L::kStageBytes >> 4;           // descriptor step between K/V stages
    uint64_t dQ = desc_kmajor_sw128(aQ);
    uint64_t dK0 = desc_kmajor_sw128(aKV);
    uint64_t dV0 = desc_mnmajor_sw128(aKV + L::kKVBytes, kKeyTile * 128, 1024);
    // S(grp) = Q(grp) K^T over D in 16-wide K-steps; the K-major SW128
    // operands hold 64 dims per 128-byte row, 8-row atoms 1 KB apart
    auto issue_s = [&](auto grp_c, uint64_t dk) {
        constexpr int grp = decltype(grp_c)::value;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = grp * L::kQGroupBytes + (kk >> 2) * (kGroupRows * 128) + (kk & 3) * 32;
            const uint32_t offk = (kk >> 2) * (kKeyTile * 128) + (kk & 3) * 32;
            mma_bf16_ss(tmem + grp * 128, dQ + (off >> 4), dk + (offk >> 4), id_s, kk > 0);
        }
        mma_commit(&s_full[grp]);
    };
    // O(grp) += P(grp) V: P from TMEM (8 columns per 16 keys), V MN-major
    // (16 keys = 16 lines of 128 B; 64-dim blocks one K/V half apart)
    auto issue_pv = [&](auto grp_c, uint64_t dv, uint32_t acc_first) {
        constexpr int grp = decltype(grp_c)::value;
#pragma unroll
        for (int kk = 0; kk < kKeyTile / 16; ++kk)
            mma_bf16_ts(tmem + 256 + grp * D, tmem + grp * 128 + kk * 8, dv + ((kk * 2048) >> 4), id_o,
                        kk > 0 ? 1u : acc_first);
        mma_commit(&o_done[grp]);
    };
    using G0 = std::integral_constant<int, 0>;
    using G1 = std::integral_constant<int, 1>;
    bool ok = mbar_wait(q_ready, 0, abort_sh);
    // prologue: S of tile 0 for every group
    if (ok) ok = mbar_wait(&k_full[0], 0, abort_sh);
    if (ok) {
        tc_fence_after();
        issue_s(G0{}, dK0);
        if constexpr (NG > 1) issue_s(G1{}, dK0);
        mma_commit(&k_empty[0]);
    }
    for (int j = 0; ok && j < ntiles; ++j) {
        // The bases pass through an empty asm each tile so that the compiler
        // forms each descriptor with one add next to its MMA instead of
        // hoisting all of them out of the loop: this warp runs on the few
        // registers the control warps keep, and hoisted descriptors spill.
        asm volatile("" : "+l"(dQ), "+l"(dK0), "+l"(dV0));
        const int st = j % kStages;
        const uint32_t ph = (uint32_t)((j / kStages) & 1);
        const int stn = (j + 1) % kStages;
        const uint32_t phn = (uint32_t)(((j + 1) / kStages) & 1);
        const bool more = j + 1 < ntiles;
        const uint64_t dv = dV0 + st * kStageStep, dkn = dK0 + stn * kStageStep;
        const uint32_t acc_first = j > 0 ? 1u : 0u;
        // This tile's V and the next tile's K land well before the P they
        // pair with: wait for them first, so that no wait but P's sits
        // between P's arrival and the MMAs it releases.  (K of tile j+1 only
        // needs S of tile j-1 to have released its stage, and V of tile j
        // only PV of tile j-2.)
        ok = mbar_wait(&v_full[st], ph, abort_sh) && (!more || mbar_wait(&k_full[stn], phn, abort_sh));
        if (!ok) break;
        // group 0: PV of this tile, then S of the next
        ok = mbar_wait(&p_full[0], j & 1, abort_sh);
        if (!ok) break;
        tc_fence_after();
        issue_pv(G0{}, dv, acc_first);
        if constexpr (NG == 1) mma_commit(&v_empty[st]);
        if (more) {
            issue_s(G0{}, dkn);
            if constexpr (NG == 1) mma_commit(&k_empty[stn]);
        }
        if constexpr (NG > 1) {
            ok = mbar_wait(&p_full[1], j & 1, abort_sh);
            if (!ok) break;
            tc_fence_after();
            issue_pv(G1{}, dv, acc_first);
            mma_commit(&v_empty[st]);
            if (more) {
                issue_s(G1{}, dkn);
                mma_commit(&k_empty[stn]);
            }
        }
    }
    if (!ok) {
        *abort_sh = 1;
        flag_error(dev_status, JSV_ERR_TIMEOUT);
    }
    int zero = 0;
    mma_commit(drain_bar);
    mbar_wait(drain_bar, 0, (volatile int *)&zero);
}

// kLpt: the work unit comes from the longest-first order (batches of 2 to
// kLptMaxReqs requests), else from the block index.  Two instantiations, so
// that the second keeps the register allocation of a kernel without the order.
template <int D, bool kLpt>
__global__ void __launch_bounds__(kAttnThreads, 1)
tree_attention_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmQ, const AttnParams prm) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    using L = AttnSmem<D>;
    constexpr int kHalves = D / 64;
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t k_full[kStages], v_full[kStages], k_empty[kStages], v_empty[kStages];
    __shared__ __align__(8) uint64_t s_full[kGroups], p_full[kGroups], o_done[kGroups], q_ready, drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ int direct_sh;              // 1: the request has one split (rows written here in bf16)
    __shared__ uint32_t anc[kRowsPerCta][kMaxTreeWords];
    __shared__ int par_sh[32 * kMaxTreeWords];

    const BatchArgs &a = prm.a;
    const int G = a.Hq / a.Hkv;
    // the work unit of this CTA: longest first for small ragged batches, else
    // by block index (x: row tile, y: split, z: request x KV head)
    int b, g, split, m0;
    Request r;
    if constexpr (kLpt) {
        __shared__ int lpt_sh[2 * kLptMaxReqs + 2];
        if (threadIdx.x < 32) {
            const int L = (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
            int ub, uloc;
            lpt_unit(prm, L, (int)threadIdx.x, lpt_sh, lpt_sh + kLptMaxReqs, ub, uloc);
            if (threadIdx.x == 0) {
                lpt_sh[2 * kLptMaxReqs] = ub;
                lpt_sh[2 * kLptMaxReqs + 1] = uloc;
            }
        }
        __syncthreads();
        b = lpt_sh[2 * kLptMaxReqs];
        if (b < 0 || !load_request(a, b, r)) return;
        const int sb = request_splits(request_tiles(r), prm.C, prm.S);
        const int R = (r.n * G + kRowsPerCta - 1) / kRowsPerCta;
        // within a request: row tile fastest, then split, then KV head (the
        // order of the block-index form, so that CTAs running side by side
        // share K/V tiles in L2)
        const int loc = lpt_sh[2 * kLptMaxReqs + 1];
        m0 = (loc % R) * kRowsPerCta;
        split = (loc / R) % sb;
        g = loc / (R * sb);
    } else {
        b = blockIdx.z / a.Hkv;
        g = blockIdx.z % a.Hkv;
        split = blockIdx.y;
        m0 = blockIdx.x * kRowsPerCta;
        // request geometry (uniform per CTA); invalid requests are flagged and skipped
        if (!load_request(a, b, r)) return;
    }
    const int rows_total = r.n * G;
    if (m0 >= rows_total) return;
    const int rows_here = min(kRowsPerCta, rows_total - m0);
    const int ngroups = rows_here > kGroupRows ? 2 : 1;     // a group with no rows is skipped

    // tile schedule for this split
    // Logical tiles: the prefix tiles, then the tree tiles; of the request's
    // Sb splits, split s takes the balanced run [total * s / Sb, total * (s + 1) / Sb).
    const int prefix_tiles = (r.P + kKeyTile - 1) / kKeyTile;
    const int P0 = r.P & ~15;                    // tree tiles start on a page boundary
    const int total_tiles = request_tiles(r);
    const int Sb = request_splits(total_tiles, prm.C, prm.S);
    if (split >= Sb) return;
    const int t_begin = (int)((long long)total_tiles * split / Sb);
    const int t_end = (int)((long long)total_tiles * (split + 1) / Sb);
    const int ntiles = t_end - t_begin;
    const int tree_tiles = max(0, t_end - max(t_begin, prefix_tiles));    // tree tiles of this split

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sKV = smem + L::kQBytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int s = 0; s < kGroups; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
            mbar_init(&o_done[s], 1);
        }
        mbar_init(&q_ready, 4 * kGroups + 1);     // softmax warps + the producer
        mbar_init(&drain_bar, 1);
        abort_sh = 0;
        direct_sh = Sb == 1 ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    // logical tile index -> first logical slot
    auto tile_slot0 = [&](int j) -> int {
        const int lj = t_begin + j;
        return lj < prefix_tiles ? lj * kKeyTile : P0 + (lj - prefix_tiles) * kKeyTile;
    };

    if (warp < kSoftmaxWarp0) {
    setmaxnreg_dec<kRegsControl>();
    if (warp == 0) {
        // ----------------------------------------------------------- producer
        // The whole warp runs the loop: lanes 0..7 look up the 8 physical pages
        // of the NEXT tile (independent loads, issued before waiting for a free
        // stage) and each issues the copies of its own page.
        if (ntiles > 0) {
            if (lane == 0) {
                // Q first: one box of 128 rows (128/G nodes x G heads) x 64 dims
                // per row group and 64-dim block; rows past the request hold
                // other nodes' (or zero-filled) queries and are never written out
                if (prm.q_tma) {
                    prefetch_tensormap(&tmQ);
                    mbar_arrive_expect_tx(&q_ready, ngroups * L::kQGroupBytes);
                    for (int grp = 0; grp < ngroups; ++grp) {
                        const int node0 = r.base + (m0 + grp * kGroupRows) / G;
#pragma unroll
                        for (int h = 0; h < kHalves; ++h)
                            tma_load_3d(sQ + grp * L::kQGroupBytes + h * (kGroupRows * 128), &tmQ, &q_ready, h * 64,
                                        g * G, node0);
                    }
                } else {
                    mbar_arrive(&q_ready);
                }
                prefetch_tensormap(&tmK);
                prefetch_tensormap(&tmV);
            }
            const int oob = a.num_pages * a.page_size;   // fully out-of-bounds slot coordinate
            const int mapped_pages = (r.P + r.n + a.page_size - 1) / a.page_size;
            // The page-table entry of page `lane` of tile j is loaded one tile
            // ahead and checked only when that tile is issued, so the load does
            // not hold up the copies of the current tile.
            auto load_page = [&](int j) -> int {         // raw entry; -2: past the mapped pages
                int page = -2;
                if (lane < kKeyTile / 16) {
                    const int lp = tile_slot0(j) / 16 + lane;
                    const long long pi = (long long)b * a.max_pages_per_req + lp;
                    if (lp < mapped_pages && JSV_IN_BOUNDS(pi, (long long)a.B * a.max_pages_per_req, a.dev_status))
                        page = __ldg(a.page_table + pi);
                }
                return page;
            };
            auto to_slot = [&](int page) -> int {        // slot coordinate of a raw entry
                if (page == -2) return oob;
                if (page >= 0 && page < a.num_pages) return page * a.page_size;
                flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
                return oob;
            };
            long long issued = 0;
            int stage = 0;
            uint32_t phase = 0;
            int page_next = load_page(0);
            bool last_v_issued = true;
            for (int j = 0; j < ntiles; ++j) {
                const int z_cur = to_slot(page_next);
                if (j + 1 < ntiles) page_next = load_page(j + 1);
                // K of a stage frees once both groups' S of its previous tile are
                // done, V once both groups' PV are
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&k_empty[stage], phase ^ 1, &abort_sh) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    if (lane == 0) {
                        abort_sh = 1;
                        flag_error(a.dev_status, JSV_ERR_TIMEOUT);
                    }
                    break;
                }
                uint8_t *sK = sKV + stage * L::kStageBytes;
                uint8_t *sV = sK + L::kKVBytes;
                if (lane == 0) mbar_arrive_expect_tx(&k_full[stage], L::kKVBytes);
                __syncwarp();
                if (lane < kKeyTile / 16) {
#pragma unroll
                    for (int h = 0; h < kHalves; ++h)
                        tma_load_3d(sK + h * (kKeyTile * 128) + lane * 2048, &tmK, &k_full[stage], h * 64, g, z_cur);
                }
                if (lane == 0) ok = mbar_wait(&v_empty[stage], phase ^ 1, &abort_sh) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    if (lane == 0) {
                        abort_sh = 1;
                        flag_error(a.dev_status, JSV_ERR_TIMEOUT);
                    }
                    last_v_issued = false;      // K of this stage is in flight, V is not
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                    break;
                }
                if (lane == 0) mbar_arrive_expect_tx(&v_full[stage], L::kKVBytes);
                __syncwarp();
                if (lane < kKeyTile / 16) {
#pragma unroll
                    for (int h = 0; h < kHalves; ++h)
                        tma_load_3d(sV + h * (kKeyTile * 128) + lane * 2048, &tmV, &v_full[stage], h * 64, g, z_cur);
                }
                ++issued;
                if (++stage == kStages) { stage = 0; phase ^= 1; }
                if (abort_sh) break;
            }
            if (lane == 0 && prm.q_tma) {
                int zero = 0;              // the Q copy has landed (long since, unless aborting)
                mbar_wait(&q_ready, 0, (volatile int *)&zero);
            }
            if (lane == 0 && abort_sh) {
                int zero = 0;
                const long long back = issued < kStages ? issued : kStages;
                int s2 = stage;
                uint32_t ph = phase;
                for (long long i = 0; i < back; ++i) {
                    if (s2 == 0) { s2 = kStages; ph ^= 1; }
                    --s2;
                    mbar_wait(&k_full[s2], ph, (volatile int *)&zero);
                    if (i > 0 || last_v_issued) mbar_wait(&v_full[s2], ph, (volatile int *)&zero);
                }
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0 && ntiles > 0) {
            const uint32_t aQ = smem_addr(sQ), aKV = smem_addr(sKV);
            if (ngroups > 1)
                attention_mma_loop<D, 2>(tmem, aQ, aKV, ntiles, k_full, v_full, k_empty, v_empty, s_full, p_full,
                                         o_done, &q_ready, &drain_bar, &abort_sh, a.dev_status);
            else
                attention_mma_loop<D, 1>(tmem, aQ, aKV, ntiles, k_full, v_full, k_empty, v_empty, s_full, p_full,
                                         o_done, &q_ready, &drain_bar, &abort_sh, a.dev_status);
        }
    }
    } else {
        setmaxnreg_inc<kRegsSoftmax>();
        // ----------------------------------------------------------- softmax
        const int grp = (warp - kSoftmaxWarp0) >> 2;  // row group of this warp
        const int sub = warp & 3;                    // TMEM lanes this warp may access
        const int grow = sub * 32 + lane;            // row within the group == TMEM lane
        const int row = grp * kGroupRows + grow;     // row within the CTA tile
        const uint32_t lane_addr = (uint32_t)(sub * 32) << 16;
        const uint32_t tS = tmem + grp * 128;
        const uint32_t tO = tmem + 256 + grp * D;
        const int et = threadIdx.x - 32 * kSoftmaxWarp0;   // 0..255
        const bool row_valid = row < rows_here;
        const int rg = m0 + row;                     // row within (b, g)
        const int node = rg / G;                     // request-local node
        const int head = g * G + rg % G;

        // With Q copied by TMA these warps take no part in it: they arrive at
        // once.  Otherwise they load Q here: rows x D bf16 in the K-major SW128
        // layout (zero rows past the end).  A thread issues a batch of loads
        // before storing any of them, so that they overlap (one memory round
        // trip per batch, not one per 16 bytes).
        if (prm.q_tma) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_ready);
        }
        constexpr int kParIters = 32 * kMaxTreeWords / (kGroups * 128);
        int pv[kParIters];
        if (tree_tiles > 0) {           // the request's parent array, for the tree mask
#pragma unroll
            for (int it = 0; it < kParIters; ++it) {
                const int i = et + it * (kGroups * 128);
                pv[it] = (i < r.n && JSV_IN_BOUNDS(r.base + i, a.total_nodes, a.dev_status))
                             ? __ldg(a.parent + r.base + i) : -1;
            }
        }
        if (!prm.q_tma) {
            constexpr int kQIters = kRowsPerCta * (D / 8) / (kGroups * 128);
            constexpr int kQBatch = kQIters < 8 ? kQIters : 8;  // loads in flight per thread
#pragma unroll
            for (int i0 = 0; i0 < kQIters; i0 += kQBatch) {
                uint4 qv[kQBatch];
#pragma unroll
                for (int it = 0; it < kQBatch; ++it) {
                    const int e = et + (i0 + it) * (kGroups * 128);
                    const int rr = e / (D / 8), c = e % (D / 8);
                    qv[it] = make_uint4(0, 0, 0, 0);
                    if (rr < rows_here) {
                        const int rgg = m0 + rr;
                        const size_t qi = ((size_t)(r.base + rgg / G) * a.Hq + g * G + rgg % G) * D + c * 8;
                        if (JSV_IN_BOUNDS(qi + 7, (long long)a.total_nodes * a.Hq * D, a.dev_status))
                            qv[it] = __ldg(reinterpret_cast<const uint4 *>(prm.q + qi));
                    }
                }
#pragma unroll
                for (int it = 0; it < kQBatch; ++it) {
                    const int e = et + (i0 + it) * (kGroups * 128);
                    const int rr = e / (D / 8), c = e % (D / 8);
                    *reinterpret_cast<uint4 *>(sQ + (rr / kGroupRows) * L::kQGroupBytes +
                                               (c >> 3) * (kGroupRows * 128) + sw128_offset(rr % kGroupRows, c & 7)) =
                        qv[it];
                }
            }
            fence_async_smem();
        }
        if (tree_tiles > 0) {
#pragma unroll
            for (int it = 0; it < kParIters; ++it) par_sh[et + it * (kGroups * 128)] = pv[it];
        }
        if (tree_tiles > 0 || !prm.q_tma) named_barrier(1, kGroups * 128);
        if (!prm.q_tma) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_ready);
        }
        // ancestor-or-self bitsets of this tile's rows (only the CTA that covers
        // the tree slots uses them), walked over the parent array in shared
        // memory; each thread reads and writes only its own row's bitset
        if (tree_tiles > 0 && row_valid) {
            for (int w = 0; w < kMaxTreeWords; ++w) anc[row][w] = 0;
            int j = node, steps = 0;
            while (j != -1) {
                if (steps++ > r.n || j >= 32 * kMaxTreeWords) {
                    flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
                    break;
                }
                anc[row][j >> 5] |= 1u << (j & 31);
                const int p = par_sh[j];
                if (j == 0 ? p != -1 : (p < 0 || p >= j)) {
                    flag_error(a.dev_status, JSV_ERR_DEVICE_INPUT);
                    break;
                }
                j = p;
            }
        }

        float m_used = -INFINITY, l = 0.f;
        const float sl2 = prm.scale_log2;
        bool ok = true;
        const int my_tiles = grp < ngroups ? ntiles : 0;
        for (int j = 0; j < my_tiles; ++j) {
            if (!mbar_wait(&s_full[grp], j & 1, &abort_sh)) ok = false;
            if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
            tc_fence_after();
            const int slot0 = tile_slot0(j);
            const bool is_tree = t_begin + j >= prefix_tiles;
            const uint32_t sbase = tS + lane_addr;
            // The whole 128-column row of S in registers: one TMEM round trip.
            uint32_t sv[kKeyTile / 32][32];
#pragma unroll
            for (int c = 0; c < kKeyTile / 32; ++c) tmem_ld_32x32b_x32(sbase + c * 32, sv[c]);
            tmem_ld_wait();
            // Masked columns (past the prefix in its last tile; non-ancestors in
            // tree tiles) become -inf.  One visibility word per 32-key chunk:
            // bit x <-> key column 32c + x.
            if (slot0 + kKeyTile > r.P) {
#pragma unroll
                for (int c = 0; c < kKeyTile / 32; ++c) {
                    const int s0 = slot0 + c * 32;
                    uint32_t vis;
                    if (!is_tree) {
                        const int cnt = r.P - s0;
                        vis = cnt >= 32 ? 0xffffffffu : (cnt <= 0 ? 0u : ((1u << cnt) - 1u));
                    } else {
                        const int j0 = s0 - r.P;         // tree node of column 32c (may be < 0)
                        vis = 0u;
                        if (row_valid && j0 > -32 && j0 < 32 * kMaxTreeWords) {
                            if (j0 < 0) {
                                vis = anc[row][0] << (-j0);
                            } else {
                                const int w = j0 >> 5;
                                const uint32_t lo = anc[row][w];
                                const uint32_t hi = (w + 1 < kMaxTreeWords) ? anc[row][w + 1] : 0u;
                                vis = __funnelshift_r(lo, hi, j0 & 31);
                            }
                        }
                    }
#pragma unroll
                    for (int x = 0; x < 32; ++x) sv[c][x] = ((vis >> x) & 1u) ? sv[c][x] : 0xff800000u;
                }
            }
            // row max of the raw scores (the scale is positive)
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < kKeyTile / 32; ++c) {
#pragma unroll
                for (int x = 0; x < 32; x += 8) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        mx[u] = fmax3(mx[u], __uint_as_float(sv[c][x + 2 * u]), __uint_as_float(sv[c][x + 2 * u + 1]));
                }
            }
            const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
            // running max with a rescale threshold
            float m_new = m_used;
            if (tmax > m_used + kRescaleThreshold || (m_used == -INFINITY && tmax > -INFINITY)) m_new = tmax;
            const float corr = (m_new == m_used) ? 1.f : fast_exp2(m_used - m_new);   // 0 when m_used = -inf

            // O holds P_0..P_{j-1} V under the old max: rescale it (rarely).  S_j
            // was issued after PV_{j-1} and its completion covers every earlier
            // product of the issuing thread, so PV_{j-1} is complete here.
            if (__any_sync(0xffffffffu, corr != 1.f) && j >= 1) {
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t ov[32];
                    tmem_ld_32x32b_x32(tO + lane_addr + c0, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * corr);
                    tmem_st_32x32b_x32(tO + lane_addr + c0, ov);
                }
                tmem_st_wait();
            }

            // probabilities (masked columns hold -inf and give 0), their sum, and
            // the bf16 P row stored into the first 64 columns of this S buffer;
            // scale, offset and row sum on packed fp32 pairs.  (Moving part of
            // the exponentials to a polynomial on the FMA pipe was measured
            // slower: this loop is bound by instruction issue, not by MUFU.)
            const float neg_m = (m_new == -INFINITY) ? 0.f : -m_new;
            const uint64_t sl2x2 = f2_pack(sl2, sl2), negmx2 = f2_pack(neg_m, neg_m);
            uint64_t ps2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
            uint32_t pk[2][32];
#pragma unroll
            for (int i = 0; i < kKeyTile / 2; ++i) {
                const int c = (2 * i) / 32, x = (2 * i) % 32;
                const uint64_t xa = f2_fma(f2_pack(__uint_as_float(sv[c][x]), __uint_as_float(sv[c][x + 1])), sl2x2, negmx2);
                float u0, u1;
                f2_unpack(xa, u0, u1);
                const uint64_t ea = f2_pack(fast_exp2(u0), fast_exp2(u1));
                ps2[i & 1] = f2_add(ps2[i & 1], ea);
                float a0, a1;
                f2_unpack(ea, a0, a1);
                pk[i / 32][i % 32] = pack_bf16x2(a0, a1);
            }
            tmem_st_32x32b_x32(sbase, pk[0]);
            tmem_st_32x32b_x32(sbase + 32, pk[1]);
            float q0, q1, q2, q3;
            f2_unpack(ps2[0], q0, q1);
            f2_unpack(ps2[1], q2, q3);
            const float psum = (q0 + q1) + (q2 + q3);
            l = l * corr + psum;
            m_used = m_new;
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[grp]);
        }

        // final partial: O (unnormalised), running max (log2 domain) and sum
        bool have_o = ok && my_tiles > 0;
        if (have_o) {
            // the last PV: every earlier one is complete (the last S came after
            // it), so the barrier is in phase my_tiles - 1 or past it and this
            // parity wait cannot alias
            if (!mbar_wait(&o_done[grp], (uint32_t)((my_tiles - 1) & 1), &abort_sh)) ok = false;
            if (__any_sync(0xffffffffu, !ok)) have_o = false;
        }
        if (!have_o) {
            m_used = -INFINITY;
            l = 0.f;
            if (!ok) {
                abort_sh = 1;
                flag_error(a.dev_status, JSV_ERR_TIMEOUT);
            }
        }
        const size_t rows = (size_t)a.total_nodes * a.Hq;
        const size_t row_id = (size_t)(r.base + min(node, r.n - 1)) * a.Hq + head;
        // A request with one split writes its rows here, normalised, in bf16;
        // otherwise this split's partial goes to the workspace in fp32.  Either
        // is written through shared memory so that global stores are whole
        // rows: each warp stages its 32 rows, half of D at a time, in its own
        // slice of this group's Q buffer (free once the group's last product
        // has completed: every product of the group precedes its last PV), XOR-
        // swizzled by row so that neither side of the transpose has bank conflicts.
        constexpr int kScrCols = D / 2;
        constexpr int kChunks = kScrCols / 4;                   // 16-byte chunks per staged row
        constexpr int kRowsPerStore = 32 / kChunks;
        float4 *scr = reinterpret_cast<float4 *>(sQ + grp * L::kQGroupBytes + sub * (32 * kScrCols * 4));
        if (have_o) tc_fence_after();
        // One pass stages half of D for the warp's 32 rows (scaled by `scale`)
        // and hands each staged 16-byte chunk to `store(row offset, column, value)`.
        auto write_rows = [&](long long my_off, float scale, auto store) {
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
                for (int c0 = 0; c0 < kScrCols; c0 += 32) {
                    uint32_t rr[32];
                    if (have_o) {
                        tmem_ld_32x32b_x32(tO + lane_addr + pass * kScrCols + c0, rr);   // warp-collective
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int x = 0; x < 32; ++x) rr[x] = 0u;
                    }
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        scr[lane * kChunks + ((c0 / 4 + x) ^ (lane & (kChunks - 1)))] =
                            make_float4(__uint_as_float(rr[4 * x]) * scale, __uint_as_float(rr[4 * x + 1]) * scale,
                                        __uint_as_float(rr[4 * x + 2]) * scale, __uint_as_float(rr[4 * x + 3]) * scale);
                }
                __syncwarp();
#pragma unroll 4
                for (int i = 0; i < 32; i += kRowsPerStore) {
                    const int wr = i + lane / kChunks, ch = lane % kChunks;
                    const long long off = __shfl_sync(0xffffffffu, my_off, wr);
                    const float4 v = scr[wr * kChunks + (ch ^ (wr & (kChunks - 1)))];
                    if (off >= 0) store(off + pass * kScrCols + ch * 4, v);
                }
                __syncwarp();
            }
        };
        if (direct_sh) {
            write_rows(row_valid ? (long long)(row_id * D) : -1ll, l > 0.f ? 1.f / l : 0.f,
                       [&](long long o, const float4 &v) {
                           if (JSV_IN_BOUNDS(o + 3, (long long)rows * D, a.dev_status))
                               *reinterpret_cast<uint2 *>(prm.out + o) = make_uint2(pack_bf16x2(v.x, v.y),
                                                                                    pack_bf16x2(v.z, v.w));
                       });
        } else {
            write_rows(row_valid ? (long long)(((size_t)split * rows + row_id) * D) : -1ll, 1.f,
                       [&](long long o, const float4 &v) {
                           if (JSV_IN_BOUNDS(o + 3, (long long)prm.S * rows * D, a.dev_status))
                               *reinterpret_cast<float4 *>(prm.ws_o + o) = v;
                       });
            const size_t mi = ((size_t)split * rows + row_id) * 2;
            if (row_valid && JSV_IN_BOUNDS(mi + 1, (long long)prm.S * rows * 2, a.dev_status)) {
                prm.ws_ml[mi + 0] = m_used;
                prm.ws_ml[mi + 1] = l;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------------------
// Split combine: one warp per (node, head) row.
// ---------------------------------------------------------------------------
// Small CTAs with at most 32 registers a thread: the combine grid becomes
// resident (and waits) while the attention kernel runs, and must leave room
// beside itself for the LM-head CTAs that start on the same SMs.
constexpr int kCombineWarps = 4;

template <int D>
__global__ void __launch_bounds__(kCombineWarps * 32, 16)
tree_attention_combine_kernel(BatchArgs a, int S_max, int C, const float *__restrict__ ws_o,
                              const float *__restrict__ ws_ml, uint16_t *__restrict__ out) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    constexpr int DPL = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.z / a.Hkv, g = blockIdx.z % a.Hkv;
    const int G = a.Hq / a.Hkv;
    const int rloc = blockIdx.x * kCombineWarps + warp;
    Request r;
    if (!load_request(a, b, r)) return;
    if (rloc >= r.n * G) return;
    const int S = request_splits(request_tiles(r), C, S_max);
    if (S == 1) return;                              // the attention kernel wrote these rows
    const int i = rloc / G, h = g * G + rloc % G, t = r.base + i;
    const size_t row_id = (size_t)t * a.Hq + h;
    const size_t rows = (size_t)a.total_nodes * a.Hq;
    // lane s holds split s's (max, sum); the merge weights come from warp
    // reductions, so the partial loads below are independent of each other
    float ms = -INFINITY, ls = 0.f;
    if (!JSV_IN_BOUNDS(row_id, rows, a.dev_status) || !JSV_IN_BOUNDS(S - 1, S_max, a.dev_status)) return;
    if (lane < S) {
        const float2 ml = *reinterpret_cast<const float2 *>(ws_ml + ((size_t)lane * rows + row_id) * 2);
        ms = ml.x;
        ls = ml.y;
    }
    float M = ls > 0.f ? ms : -INFINITY;
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, sh));
    const float cw = ls > 0.f ? exp2f(ms - M) : 0.f;
    float L = ls * cw;
#pragma unroll
    for (int sh = 16; sh > 0; sh >>= 1) L += __shfl_xor_sync(0xffffffffu, L, sh);
    float o[DPL];
#pragma unroll
    for (int x = 0; x < DPL; ++x) o[x] = 0.f;
#pragma unroll 4
    for (int s = 0; s < S; ++s) {
        const float c = __shfl_sync(0xffffffffu, cw, s);
        if (c == 0.f) continue;
        const float *po = ws_o + ((size_t)s * rows + row_id) * D + lane * DPL;
        if constexpr (DPL == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(po);
            o[0] = fmaf(c, v.x, o[0]);
            o[1] = fmaf(c, v.y, o[1]);
            o[2] = fmaf(c, v.z, o[2]);
            o[3] = fmaf(c, v.w, o[3]);
        } else {
#pragma unroll
            for (int x = 0; x < DPL; ++x) o[x] = fmaf(c, po[x], o[x]);
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    uint16_t *op = out + row_id * D + lane * DPL;
#pragma unroll
    for (int x = 0; x < DPL; ++x) {
        __nv_bfloat16 hb = __float2bfloat16_rn(o[x] * inv);
        op[x] = *reinterpret_cast<uint16_t *>(&hb);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
// Key tiles of the largest request the batch may hold (a bound on every
// request's prefix + tree tiles).
static int max_request_tiles(const BatchArgs &a) {
    return (a.max_prefix + kKeyTile - 1) / kKeyTile + (a.max_nodes + 15 + kKeyTile - 1) / kKeyTile;
}

static int attention_splits(const BatchArgs &a) {
    // Choose S, the splits of the largest request, to minimise an estimate of
    // the kernel time in tile periods (about 2.3 us each): waves(S) * (kFixed
    // + ceil(total / S)) plus, per split, the write and read of its fp32
    // partial at about 6 TB/s, where total = prefix tiles + tree tiles of the
    // largest request, a wave is one CTA per SM and kFixed covers set-up, the
    // first loads and the partial write of a CTA.  (Shorter requests take
    // proportionally fewer splits, so the estimate is an upper bound.)
    const int G = a.Hq / a.Hkv;
    const int mtiles = (a.max_nodes * G + kRowsPerCta - 1) / kRowsPerCta;
    const long long units = (long long)a.B * a.Hkv * mtiles;
    const int total = max_request_tiles(a);
    const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
    const double kFixed = 3.0, kTileUs = 2.3;
    const double comb = (double)a.total_nodes * a.Hq * (a.D + 2) * 4.0 * 2.0 / 6.0e6 / kTileUs;   // per split
    int best = 1;
    double best_cost = 1e300;
    for (int s = 1; s <= 32 && s <= total; ++s) {
        const long long waves = (units * s + sms - 1) / sms;
        const double cost = (double)waves * (kFixed + (double)((total + s - 1) / s)) + (s > 1 ? s * comb : 0.0);
        if (cost < best_cost - 1e-9) { best_cost = cost; best = s; }
    }
    return best;
}

size_t attention_workspace_bytes(const BatchArgs &a) {
    const size_t rows = (size_t)a.total_nodes * a.Hq;
    const int S = attention_splits(a);
    return S > 1 ? (size_t)S * rows * ((size_t)a.D + 2) * sizeof(float) : 0;   // one split: no partials
}

template <int D>
static cudaError_t launch_d(const BatchArgs &a, const uint16_t *q, const uint16_t *k_cache,
                            const uint16_t *v_cache, float scale, uint16_t *out, void *ws, cudaStream_t st) {
    using Lt = AttnSmem<D>;
    const int S = attention_splits(a);
    const int G = a.Hq / a.Hkv;
    const size_t rows = (size_t)a.total_nodes * a.Hq;
    AttnParams prm;
    prm.a = a;
    prm.q = q;
    prm.out = out;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.S = S;
    prm.C = (max_request_tiles(a) + S - 1) / S;
    prm.ws_o = S > 1 ? static_cast<float *>(ws) : nullptr;
    prm.ws_ml = S > 1 ? prm.ws_o + (size_t)S * rows * D : nullptr;

    CUtensorMap tmK, tmV, tmQ;
    memset(&tmQ, 0, sizeof(tmQ));
    prm.q_tma = (kGroupRows % G == 0 &&
                 encode_tensor_map_3d(&tmQ, q, D, a.Hq, a.total_nodes, (uint64_t)D * 2, (uint64_t)a.Hq * D * 2, 64,
                                      G, kGroupRows / G))
                    ? 1
                    : 0;
    const uint64_t slots = (uint64_t)a.num_pages * a.page_size;
    if (!encode_tensor_map_3d(&tmK, k_cache, D, a.Hkv, slots, (uint64_t)D * 2, (uint64_t)a.Hkv * D * 2, 64, 1, 16))
        return cudaErrorInvalidValue;
    if (!encode_tensor_map_3d(&tmV, v_cache, D, a.Hkv, slots, (uint64_t)D * 2, (uint64_t)a.Hkv * D * 2, 64, 1, 16))
        return cudaErrorInvalidValue;
    const size_t smem = (size_t)Lt::kTotal + 1024;
    auto set_attrs = [&](auto kernel) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        return e;
    };
    static PerDeviceOnce attr_once;
    cudaError_t ae = attr_once.run([&]() {
        cudaError_t e = set_attrs(tree_attention_tc_kernel<D, false>);
        return e == cudaSuccess ? set_attrs(tree_attention_tc_kernel<D, true>) : e;
    });
    if (ae != cudaSuccess) return ae;
    // Longest-first order when each CTA takes a request's whole key range
    // (S = 1), so that the longest requests do not start last; with several
    // splits the per-request split counts already even the units out, and the
    // order's set-up and register cost is not paid.
    const bool lpt = S == 1 && a.B > 1 && a.B <= kLptMaxReqs;
    auto kernel = lpt ? tree_attention_tc_kernel<D, true> : tree_attention_tc_kernel<D, false>;
    dim3 grid((a.max_nodes * G + kRowsPerCta - 1) / kRowsPerCta, S, a.B * a.Hkv);
    cudaError_t le = launch_pdl(kernel, grid, dim3(kAttnThreads), smem, st, tmK, tmV, tmQ, prm);
    if (le != cudaSuccess) {
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kernel) == cudaSuccess)
            note_launch_failure("tree attention", fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes,
                                fa.maxDynamicSharedSizeBytes, kAttnThreads, smem);
        return le;
    }
    if (S == 1) {                 // every row was written by the attention kernel
        count_launches(1);
        return cudaSuccess;
    }
    dim3 cgrid((a.max_nodes * G + kCombineWarps - 1) / kCombineWarps, 1, a.B * a.Hkv);
    static PerDeviceOnce carve;
    le = prefer_max_shared(tree_attention_combine_kernel<D>, carve);
    if (le != cudaSuccess) return le;
    le = launch_pdl(tree_attention_combine_kernel<D>, cgrid, dim3(kCombineWarps * 32), 0, st, a, S, prm.C,
                    (const float *)prm.ws_o, (const float *)prm.ws_ml, out);
    count_launches(2);
    return le;
}

cudaError_t launch_tree_attention(const BatchArgs &a, const uint16_t *q, const uint16_t *k_cache,
                                  const uint16_t *v_cache, float scale, uint16_t *out, void *ws,
                                  cudaStream_t st) {
    if (a.D == 128) return launch_d<128>(a, q, k_cache, v_cache, scale, out, ws, st);
    return launch_d<64>(a, q, k_cache, v_cache, scale, out, ws, st);
}

}  // namespace jsv
