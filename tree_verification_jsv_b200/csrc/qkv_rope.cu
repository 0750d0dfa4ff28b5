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
// memory; then each warp takes 8 of the slice's nodes and each lane 4
// consecutive rows of one of them, rotates them against their partners and
// writes 8 bytes of bf16 to q or to the cache (a warp covers a node's 128
// rows with 256 contiguous bytes).
// When (tile, node group) CTAs alone would leave SMs idle (one 64-node tree:
// 48 tiles for Qwen3-8B), a cluster of up to four CTAs splits K: each reduces
// its share of d into its own TMEM and, once the first CTA's ring is idle,
// stores every 32-node slice of its partial into a slot of its own in the
// first CTA's shared memory (distributed shared memory; bounded mbarrier
// handshakes: ring idle on the others, one ready per slice on the first CTA),
// and the first CTA adds the slots to its own partial slice by slice and runs
// the epilogue.
// Under programmatic dependent launch the producer issues the first ring's
// worth of W copies before it waits for the previous launch: W is a weight
// that no call of this library writes, while x, the batch geometry and the
// cache rows written here are read or written only after the wait.
#include "jsv_internal.cuh"
#include "sm100.cuh"

#include <map>
#include <mutex>
#include <tuple>

namespace jsv {

using namespace sm100;

namespace {

constexpr int kQThreads = 192;
constexpr int kQMaxSplit = 4;                    // CTAs of a cluster splitting K
constexpr int kQMaxSlices = 8;                   // 32-node slices of a group (at most 256 nodes)
constexpr int kQMaxStages = 6;
constexpr int kQTileM = 128;
constexpr int kQKChunk = 64;
constexpr uint32_t kQStageA = kQTileM * 128;
// The ring may take the shared memory the other arrays leave (the epilogue's
// slice buffer and the K-split slots reuse the ring once the accumulator is
// complete), up to six
// stages: groups of 256 nodes (16 KB of W + 32 KB of x a stage) get four
// stages instead of three, measured 50.0 -> 47.0 us for one 256-node tree of
// Qwen3-8B shapes; more than six stages slowed the 64-node case (nine:
// 26.8 -> 28.6 us), so the cap keeps it at six.
constexpr int kQSmemBudget = 216 * 1024;
// A smaller ring that lets two CTAs share an SM, so that clusters of three
// find room in one resident wave (about 5 KB of static shared memory a CTA).
constexpr int kQSmemBudgetShared = 72 * 1024;
constexpr int kQMaxWalk = 512 + 256;             // parents a group's depth walks can visit

struct QkvParams {
    BatchArgs a;
    int d, rows_total, kchunks, group_nodes, box_rows, stages;
    int ksplit;        // CTAs of a cluster splitting K (1: no cluster)
    uint32_t stage_bytes;
    const float *cos, *sin;
    int max_pos;
    uint16_t *q, *k_cache, *v_cache;
};

// Hint: bring the 128-byte line holding global address p into L2.
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

// Store to a shared::cluster address (from cluster_addr).
__device__ __forceinline__ void st_shared_cluster_b32(uint32_t cluster_addr, uint32_t v) {
    asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// 16-byte read-only global load issued where it stands (not moved by the
// compiler), so that its latency overlaps the code that follows.
__device__ __forceinline__ float4 ld_global_nc_f4(const float *p) {
    float4 v;
    asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(reinterpret_cast<uint64_t>(p)));
    return v;
}

// Two floats rounded to nearest-even bf16 with one packed conversion; lo in
// the low half.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__global__ void __launch_bounds__(kQThreads, 2)
qkv_rope_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                const QkvParams p) {
    pdl_allow_dependents();
    extern __shared__ uint8_t dsmem[];
    __shared__ __align__(8) uint64_t full_bar[kQMaxStages], empty_bar[kQMaxStages], accf_bar, drain_bar;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int ep_fail;
    // slice_ready[sl] (first CTA): the other CTAs' partials of slice sl have
    // landed; ring_idle (other CTAs): the first CTA's ring, which holds the
    // slots, is idle.  One phase each.
    __shared__ __align__(8) uint64_t slice_ready[kQMaxSlices], ring_idle;
    __shared__ int s_pos[256], s_row[256];
    __shared__ int s_par[kQMaxWalk];

    const BatchArgs &a = p.a;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    // Epilogue buffers over the start of the ring, used once the first CTA's
    // last MMA has completed (every stage consumed, no copy in flight): one
    // 32-node slice, a row of 128 tile rows per node, then, in the first CTA,
    // a slot for every (other CTA q, slice) pair (the same offsets in every
    // CTA), so the other CTAs store all their slices as soon as the ring is
    // idle (the launch only splits K where the ring has room for them).
    float (*tile)[kQTileM] = reinterpret_cast<float (*)[kQTileM]>(smem);
    const int nslices = (p.group_nodes + 31) / 32;
    auto recv = [&](int q, int sl) {
        return reinterpret_cast<float (*)[kQTileM]>(smem + (size_t)(1 + (q - 1) * nslices + sl) * sizeof(float) * 32 *
                                                              kQTileM);
    };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // K split: CTA ks of the cluster reduces K-chunks [kc0, kc1); the first
    // CTA adds the others' partials and runs the epilogue
    const int ks = p.ksplit > 1 ? (int)cluster_ctarank() : 0;
    const int kc0 = p.kchunks * ks / p.ksplit, kc1 = p.kchunks * (ks + 1) / p.ksplit;
    const int row0 = (blockIdx.x / p.ksplit) * kQTileM;
    const int node0 = blockIdx.y * p.group_nodes;
    const int in_group = min(p.group_nodes, a.total_nodes - node0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&accf_bar, 1);
        mbar_init(&drain_bar, 1);
        for (int sl = 0; sl < kQMaxSlices; ++sl)                         // the other CTAs' epilogue warps
            mbar_init(&slice_ready[sl], 4 * (p.ksplit > 1 ? p.ksplit - 1 : 1));
        mbar_init(&ring_idle, 4);                                        // the first CTA's epilogue warps
        abort_sh = 0;
        ep_fail = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    if (p.ksplit > 1) cluster_sync();            // every CTA's barriers initialised
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    if (warp >= 2) pdl_wait_predecessor();       // the epilogue reads the geometry and writes q and the cache

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmW);
            prefetch_tensormap(&tmX);
            const uint32_t tx = kQStageA + (uint32_t)p.box_rows * 128;
            // the first ring's W copies (fresh stages need no wait), then the
            // wait for the previous launch, then their x copies
            const int npre = min(p.stages, kc1 - kc0);
            for (int i = 0; i < npre; ++i) {
                mbar_arrive_expect_tx(&full_bar[i], tx);
                tma_load_2d(smem + (size_t)i * p.stage_bytes, &tmW, &full_bar[i], (kc0 + i) * kQKChunk, row0);
            }
            pdl_wait_predecessor();
            for (int i = 0; i < npre; ++i)
                tma_load_2d(smem + (size_t)i * p.stage_bytes + kQStageA, &tmX, &full_bar[i], (kc0 + i) * kQKChunk,
                            node0);
            int stage = npre == p.stages ? 0 : npre;
            uint32_t phase = npre == p.stages ? 1u : 0u;
            long long issued = npre;
            for (int kc = kc0 + npre; kc < kc1; ++kc) {
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
            for (int kc = kc0; kc < kc1; ++kc) {
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
                                (kc > kc0 || kk > 0) ? 1u : 0u);
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
        auto request_of = [&](int t) {               // node_offsets is sorted
            int lo = 0, hi = a.B - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (a.node_offsets[mid] <= t) lo = mid; else hi = mid - 1;
            }
            return lo;
        };
        // The depth walks only visit nodes of the requests that overlap this
        // group, [first such request's base, node0 + in_group): at most 512 +
        // 256 entries, staged in shared memory with one coalesced load.
        const int wbase = a.node_offsets[request_of(node0)];
        const int wcount = node0 + in_group - wbase;
        const bool staged = wbase >= 0 && wcount > 0 && wcount <= kQMaxWalk;
        if (staged)
            for (int i = et; i < wcount; i += 128) s_par[i] = __ldg(a.parent + wbase + i);
        named_barrier(1, 128);
        for (int c = et; c < in_group; c += 128) {
            const int t = node0 + c;
            const int lo = request_of(t);
            Request req;
            int pos = -1, row = -1;
            if (load_request(a, lo, req)) {
                int j = t - req.base, dep = 0, steps = 0;
                bool ok = true;
                while (j > 0) {
                    const int gi = req.base + j;
                    int pj = -1;
                    if (staged && gi >= wbase && gi < wbase + wcount) pj = s_par[gi - wbase];
                    else if (JSV_IN_BOUNDS(gi, a.total_nodes, a.dev_status)) pj = a.parent[gi];
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

        const int qrows = a.Hq * a.D, krows = a.Hkv * a.D, half = a.D / 2;
        // While the main loop runs, the rotary tables' rows at this group's
        // positions go to L2 (only the first CTA of a cluster rotates, and
        // only tiles with Q or K rows).
        if (ks == 0 && row0 < qrows + krows) {
            for (int c = et; c < in_group; c += 128) {
                const int pos = s_pos[c];
                if (pos < 0 || pos >= p.max_pos) continue;
                for (int off = 0; off < half; off += 32) {          // 128-byte lines
                    prefetch_l2(p.cos + (size_t)pos * half + off);
                    prefetch_l2(p.sin + (size_t)pos * half + off);
                }
            }
        }

        if (!mbar_wait(&accf_bar, 0, &abort_sh)) {
            abort_sh = 1;
            flag_error(a.dev_status, JSV_ERR_TIMEOUT);
            ep_fail = 1;
        }
        named_barrier(1, 128);
        if (!ep_fail) {
            tc_fence_after();
            // The first CTA's ring is idle from here on: the other CTAs may
            // store their partials into its slots.
            if (ks == 0 && p.ksplit > 1 && lane == 0)
                for (int q = 1; q < p.ksplit; ++q) mbar_arrive_cluster(cluster_addr(&ring_idle, (uint32_t)q));
            // Each warp takes 8 of a slice's 32 nodes (x = sub + 4k) and each
            // lane 4 consecutive rows of the tile, so a warp writes a node's
            // 128 rows as 256 contiguous bytes with one 8-byte store a lane.
            const int q0 = lane * 4;                        // tile rows q0 .. q0 + 3
            const int g0 = row0 + q0;
            const int kq = g0 < qrows ? 0 : (g0 < qrows + krows ? 1 : 2);   // Q, K, V
            const int hq = kq == 0 ? g0 : (kq == 1 ? g0 - qrows : g0 - qrows - krows);
            const int headq = hq / a.D, oq = hq % a.D, iq = oq % half;
            const bool qvalid = g0 + 3 < p.rows_total;
            bool ring_ok = false;                   // (other CTAs) the first CTA's ring was seen idle
            for (int c0 = 0, sl = 0; c0 < in_group; c0 += 32, ++sl) {
                // the slice's cos/sin loads go out first, so their latency
                // overlaps the accumulator read and the cross-CTA sum
                float4 cs[8], sn[8];
                if (ks == 0) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int c = c0 + sub + 4 * k;
                        const int pos = c < in_group ? s_pos[c] : -1;
                        cs[k] = make_float4(1.f, 1.f, 1.f, 1.f);
                        sn[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (kq < 2 && qvalid && pos >= 0 &&
                            JSV_IN_BOUNDS((long long)pos * half + iq + 3, (long long)p.max_pos * half, a.dev_status)) {
                            cs[k] = ld_global_nc_f4(p.cos + (size_t)pos * half + iq);
                            sn[k] = ld_global_nc_f4(p.sin + (size_t)pos * half + iq);
                        }
                    }
                }
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem + lane_addr + (uint32_t)c0, v);
                tmem_ld_wait();
                if (ks > 0) {
                    // store this partial into its slot of the first CTA once that
                    // CTA's ring is idle (waited for before the first slice); the
                    // first CTA reads it locally.  A warp whose wait runs out (in
                    // any lane) skips its stores from then on (no named barrier on
                    // this path).
                    if (sl == 0) ring_ok = __all_sync(0xffffffffu, mbar_wait_cluster(&ring_idle, 0u, &abort_sh));
                    if (!ring_ok) {
                        if (lane == 0) flag_error(a.dev_status, JSV_ERR_TIMEOUT);
                        continue;
                    }
                    const uint32_t dst = cluster_addr(&recv(ks, sl)[0][r], 0);
#pragma unroll
                    for (int x = 0; x < 32; ++x) st_shared_cluster_b32(dst + (uint32_t)(x * kQTileM * 4), v[x]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(cluster_addr(&slice_ready[sl], 0));
                    continue;
                }
                if (p.ksplit > 1) {
                    // add the other CTAs' partials of this slice in rank (K) order.
                    // A warp whose wait runs out raises ep_fail and still takes the
                    // slice's named barriers; every warp then leaves after the
                    // first of them.
                    if (__all_sync(0xffffffffu, mbar_wait_cluster(&slice_ready[sl], 0u, &abort_sh))) {
                        for (int q = 1; q < p.ksplit; ++q) {
                            const float(*pq)[kQTileM] = recv(q, sl);
#pragma unroll
                            for (int x = 0; x < 32; ++x) v[x] = __float_as_uint(__uint_as_float(v[x]) + pq[x][r]);
                        }
                    } else if (lane == 0) {
                        flag_error(a.dev_status, JSV_ERR_TIMEOUT);
                        ep_fail = 1;
                    }
                }
#pragma unroll
                for (int x = 0; x < 32; ++x) tile[x][r] = __uint_as_float(v[x]);
                named_barrier(1, 128);
                if (ep_fail) break;                         // every epilogue warp sees the same flag here
                // One epilogue warp per SM sub-partition, so nothing hides a
                // dependent chain: every read of a half-slice goes out before any
                // use, and only the stores are predicated.
                const float sg = oq < half ? -1.f : 1.f;             // rotate-half sign
                uint16_t *const base = kq == 0 ? p.q : (kq == 1 ? p.k_cache : p.v_cache);
                const long long dn = kq == 0 ? (long long)a.total_nodes * a.Hq * a.D
                                             : (long long)a.num_pages * a.page_size * a.Hkv * a.D;
#pragma unroll
                for (int h4 = 0; h4 < 8; h4 += 4) {
                    int row_of[4];
                    float4 vv[4], pp[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int x = sub + 4 * (h4 + k), c = c0 + x;
                        const bool ok = qvalid && c < in_group && s_pos[c] >= 0 && s_row[c] >= 0;
                        row_of[k] = !ok ? -1 : (kq == 0 ? node0 + c : s_row[c]);
                        vv[k] = *reinterpret_cast<const float4 *>(&tile[x][q0]);
                        pp[k] = *reinterpret_cast<const float4 *>(&tile[x][q0 ^ half]);
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        float4 v = vv[k];
                        if (kq < 2) {
                            const float4 c4 = cs[h4 + k], s4 = sn[h4 + k], pv = pp[k];
                            v.x = fmaf(v.x, c4.x, sg * pv.x * s4.x);
                            v.y = fmaf(v.y, c4.y, sg * pv.y * s4.y);
                            v.z = fmaf(v.z, c4.z, sg * pv.z * s4.z);
                            v.w = fmaf(v.w, c4.w, sg * pv.w * s4.w);
                        }
                        if (row_of[k] < 0) continue;
                        uint2 pk;
                        pk.x = pack_bf16x2_rn(v.x, v.y);
                        pk.y = pack_bf16x2_rn(v.z, v.w);
                        // q row: the node; cache row: its physical slot
                        const long long di = ((long long)row_of[k] * (kq == 0 ? a.Hq : a.Hkv) + headq) * a.D + oq;
                        if (!JSV_IN_BOUNDS(di + 3, dn, a.dev_status)) continue;
                        *reinterpret_cast<uint2 *>(base + di) = pk;
                    }
                }
                named_barrier(1, 128);
            }
        }
    }

    __syncwarp();
    tc_fence_before();
    if (p.ksplit > 1) cluster_sync();            // no CTA leaves while its partial may still be read
    else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// Clusters of `cfg` that fit on the current device at once, remembered per
// (device, cluster size, dynamic shared memory): the occupancy query costs
// host time that every call would otherwise pay.  Failed queries are not
// remembered.
int active_clusters(cudaLaunchConfig_t &cfg, int ks) {
    static std::mutex mu;
    static std::map<std::tuple<int, int, size_t>, int> known;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const auto key = std::make_tuple(dev, ks, cfg.dynamicSmemBytes);
    {
        std::lock_guard<std::mutex> lock(mu);
        const auto it = known.find(key);
        if (it != known.end()) return it->second;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, qkv_rope_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    std::lock_guard<std::mutex> lock(mu);
    known[key] = n;
    return n;
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
    auto stages_for = [&](int budget) { return min(kQMaxStages, budget / (int)p.stage_bytes); };
    p.stages = stages_for(kQSmemBudget);
    if ((size_t)p.stages * p.stage_bytes < 2 * 32 * kQTileM * sizeof(float)) return cudaErrorInvalidValue;
    p.cos = rope_cos;
    p.sin = rope_sin;
    p.max_pos = max_pos;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.ksplit = 1;

    CUtensorMap tmW, tmX;
    if (!encode_tensor_map_2d(&tmW, w_qkv, (uint64_t)d, (uint64_t)p.rows_total, (uint64_t)d * 2, kQKChunk, kQTileM))
        return cudaErrorInvalidValue;
    if (!encode_tensor_map_2d(&tmX, x, (uint64_t)d, (uint64_t)a.total_nodes, (uint64_t)d * 2, kQKChunk, p.box_rows))
        return cudaErrorInvalidValue;
    size_t smem = (size_t)p.stages * p.stage_bytes + 1024;
    static PerDeviceOnce attr_once;
    cudaError_t ae = attr_once.run([]() {
        cudaError_t e = cudaFuncSetAttribute(qkv_rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kQSmemBudget + 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(qkv_rope_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        return e;
    });
    if (ae != cudaSuccess) return ae;
    const int tiles = (p.rows_total + kQTileM - 1) / kQTileM;
    const int groups = (a.total_nodes + p.group_nodes - 1) / p.group_nodes;
    // Too few (tile, group) CTAs to stream the weight with every SM: split K
    // over a cluster of up to four CTAs (each keeping at least four chunks),
    // as many as the SMs and the resident clusters allow.  Clusters are placed
    // within one GPC, so a split that does not fit in one wave with the full
    // ring is tried again with the smaller ring, which lets two CTAs share an
    // SM; more CTAs streaming W beat a deeper ring per CTA.
    const int sms = device_sm_count();
    int ks = 1;
    while (ks < kQMaxSplit && (long long)tiles * groups * (ks + 1) <= sms && p.kchunks / (ks + 1) >= 4) ++ks;
    bool placed = false;
    for (; ks > 1 && !placed; --ks) {
        for (int budget : {kQSmemBudget, kQSmemBudgetShared}) {
            const int st_n = stages_for(budget);
            // the ring holds the slice buffer and a slot per (other CTA, slice)
            const size_t slots = 1 + (size_t)(ks - 1) * ((p.group_nodes + 31) / 32);
            if (st_n < 2 || (size_t)st_n * p.stage_bytes < slots * 32 * kQTileM * sizeof(float)) continue;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(tiles * ks, groups);
            cfg.blockDim = dim3(kQThreads);
            cfg.dynamicSmemBytes = (size_t)st_n * p.stage_bytes + 1024;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = ks;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            const int n = active_clusters(cfg, ks);
            if ((long long)n >= (long long)tiles * groups) {     // one resident wave
                p.stages = st_n;
                smem = cfg.dynamicSmemBytes;
                placed = true;
                break;
            }
        }
        if (placed) break;
    }
    if (!placed) ks = 1;
    p.ksplit = ks;
    dim3 grid(tiles * ks, groups);
    cudaError_t e = ks > 1 ? launch_pdl_cluster(qkv_rope_kernel, grid, dim3(kQThreads), smem, st, ks, tmW, tmX, p)
                           : launch_pdl(qkv_rope_kernel, grid, dim3(kQThreads), smem, st, tmW, tmX, p);
    count_launches(1);
    return e;
}

}  // namespace jsv
