// Budgeted draft-tree construction by cumulative log-probability.
//
// JetSpec README, "Evaluation": the default tree construction (accum_logp)
// keeps a breadth-first tree by cumulative log-probability under depth,
// width and budget.  Reading: the draft head gives, per depth m = 1..D, its
// top-k tokens with log-probabilities sorted in descending order; a node is
// a rank path, scored by the fp32 running sum of its edge log-probs (added
// root to leaf); the tree is the `budget` best nodes under
//     score descending, depth ascending, rank path (lexicographic) ascending,
// which is ancestor- and sibling-closed, emitted breadth-first.
//
// One CTA of 16 warps per request, no sorting and no heap:
//  1. tau, the budget-th best score, by a 16-way search over the fp32 order
//     (each round every warp tests one threshold, ~8 rounds instead of 32;
//     a round costs one warp's expansion latency, so 16 warps measured
//     faster than 32 or 8):
//     count(x) = #nodes with score >= x comes from a level-by-level expansion
//     that stops as soon as it reaches the budget (children of a node are
//     scanned in rank order and stop at the first one below x, since the
//     log-probs are sorted);
//  2. one more level-by-level expansion materialises the nodes with score
//     > tau plus the first (budget - #{score > tau}) nodes with score == tau
//     in breadth-first order.  Within a level, breadth-first order is the
//     lexicographic order of the rank paths, so this is exactly the tie rule.
// The expansion writes nodes level by level, children of each parent in
// rank order, parents in breadth-first order: the output is breadth-first.
#include "jsv_internal.cuh"

#include <math.h>

namespace jsv {

constexpr int kTreeMaxBudget = 512;
constexpr int kTreeMaxWidth = 32;
constexpr int kTreeMaxDepth = 32;

struct TreeArgs {
    const float *logp;          // [B][D][k]
    const int32_t *topk_tokens; // [B][D][k]
    const int32_t *root_token;  // [B]
    int B, D, k, budget;
    int32_t *parent, *tokens, *depth;   // [B][budget]
    float *score;                       // [B][budget] or NULL
    int32_t *num_nodes;                 // [B]
    int32_t *status;
};

__device__ __forceinline__ uint32_t f2ord(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

constexpr int kTreeWarpsLog2 = 4;
constexpr int kTreeWarps = 1 << kTreeWarpsLog2;  // warps a request: one threshold each per round
constexpr int kTreeLevel = kTreeMaxBudget + kTreeMaxWidth;

struct TreeSmem {
    float lp[kTreeMaxDepth][kTreeMaxWidth];
    float nscore[kTreeMaxBudget];
    int32_t nparent[kTreeMaxBudget];
    uint8_t nrank[kTreeMaxBudget];
    uint8_t ndepth[kTreeMaxBudget];
    int res[kTreeWarps];
    int cnt[kTreeWarps];                       // their counts (exact below the budget)
    uint32_t tw[kTreeWarps];                   // the thresholds of a search round
    uint32_t lo, hi;
    int bad, take_all, nodes, vfirst, hi_count;
};

// Number of nodes with score >= x, capped at `cap` (exits as soon as it is
// reached).  One warp, with its own two level buffers; the result is uniform.
// Only the count and the set of next-level scores matter here (not their
// order), so each 32-node chunk of a level is expanded one child rank at a
// time with a ballot: a lane whose rank-r child falls below x has no later
// passing child (the log-probs are sorted), and a rank that no lane passes
// ends the chunk.
__device__ int count_ge(const TreeSmem &sm, float *cur, float *nxt, int D, int k, float x, int cap, int lane) {
    if (lane == 0) cur[0] = 0.f;
    __syncwarp();
    int ncur = 1, total = 1;
    if (total >= cap) return cap;
    const unsigned lt = (1u << lane) - 1u;
    for (int m = 0; m < D && ncur > 0; ++m) {
        int base = 0;
        for (int c0 = 0; c0 < ncur; c0 += 32) {
            const int i = c0 + lane;
            const bool live = i < ncur;
            const float s = live ? cur[i] : 0.f;
            for (int r = 0; r < k; ++r) {
                const float sc = __fadd_rn(s, sm.lp[m][r]);
                const unsigned b = __ballot_sync(0xffffffffu, live && sc >= x);
                if (b == 0u) break;
                const int nb = __popc(b);
                if (total + base + nb >= cap) return cap;
                if ((b >> lane) & 1u) nxt[base + __popc(b & lt)] = sc;
                base += nb;
            }
        }
        __syncwarp();
        total += base;
        ncur = base;
        float *t = cur; cur = nxt; nxt = t;
    }
    return total;
}

__global__ void __launch_bounds__(32 * kTreeWarps)
accum_logp_tree_kernel(TreeArgs a) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    __shared__ TreeSmem sm;
    extern __shared__ float lvl_all[];             // [kTreeWarps][2][kTreeLevel]
    const int b = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float *lvl0 = lvl_all + (size_t)warp * 2 * kTreeLevel, *lvl1 = lvl0 + kTreeLevel;
    const int k = a.k, budget = a.budget;
    int32_t *o_par = a.parent + (size_t)b * budget;
    int32_t *o_tok = a.tokens + (size_t)b * budget;
    int32_t *o_dep = a.depth + (size_t)b * budget;
    float *o_sc = a.score ? a.score + (size_t)b * budget : nullptr;

    // stage and validate the log-probs: finite or -inf, <= 0, non-increasing per depth
    if (threadIdx.x == 0) sm.bad = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < a.D * k; e += blockDim.x) {
        const float v = a.logp[((size_t)b * a.D) * k + e];
        if (!(v <= 0.f) && !(v == -INFINITY)) sm.bad = 1;
        sm.lp[e / k][e % k] = v;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.D * k; e += blockDim.x) {
        const int m = e / k, r = e % k;
        if (r > 0 && !(sm.lp[m][r] <= sm.lp[m][r - 1])) sm.bad = 1;
    }
    __syncthreads();
    int D = a.D;
    if (sm.bad) {
        if (threadIdx.x == 0) flag_error(a.status, JSV_ERR_DEVICE_INPUT);
        D = 0;    // emit the root alone
    }

    // 1. tau: the largest x with count(x) >= budget.  Invariant count(lo) >=
    //    budget > count(hi) over the fp32 order; each round warp w tests a
    //    threshold t_w (t_0 = lo, non-decreasing in w) and the interval
    //    shrinks to the last passing threshold and the next (count is
    //    non-increasing in x).  The first round spaces the thresholds evenly
    //    in value over [smin, 0], where smin is the lowest score a node can
    //    have; later rounds evenly over the fp32 order, lo + (hi - lo) w / W.
    if (threadIdx.x == 0) {
        sm.lo = f2ord(-INFINITY);
        sm.hi = f2ord(0.f) + 1u;
        sm.take_all = 0;
        sm.vfirst = 0;
        sm.hi_count = 0;                         // no node scores above 0
    }
    __syncthreads();
    const bool search = budget > 1 && D > 0;
    if (search && warp == 0) {
        const int all = count_ge(sm, lvl0, lvl1, D, k, -INFINITY, budget, lane);
        if (lane == 0) sm.take_all = all < budget;   // the whole candidate tree fits the budget
    }
    __syncthreads();
    if (search && !sm.take_all) {
        // smin: every depth's smallest log-prob summed in fp32 in the order
        // the expansion adds them; no node scores lower, so count(smin) is the
        // whole candidate tree (at least the budget, as take_all is false)
        if (threadIdx.x == 0) {
            float smin = 0.f;
            for (int m = 0; m < D; ++m) smin = __fadd_rn(smin, sm.lp[m][k - 1]);
            if (smin > -INFINITY) {
                sm.lo = f2ord(smin);
                sm.vfirst = 1;
            }
        }
        __syncthreads();
        while (sm.hi - sm.lo > 1u) {
            const uint32_t lo = sm.lo, hi = sm.hi;
            uint32_t t;
            if (sm.vfirst) {
                const float v = ord2f(lo) * (1.f - (float)warp / (float)kTreeWarps);    // hi is just above 0
                t = warp == 0 ? lo : min(max(f2ord(v), lo + 1u), hi - 1u);
            } else {
                t = lo + (uint32_t)(((unsigned long long)(hi - lo) * (unsigned)warp) >> kTreeWarpsLog2);
            }
            const int c = warp == 0 ? budget : count_ge(sm, lvl0, lvl1, D, k, ord2f(t), budget, lane);
            if (lane == 0) {
                sm.res[warp] = c >= budget;
                sm.cnt[warp] = c;
                sm.tw[warp] = t;
            }
            __syncthreads();
            if (warp == 0) {
                // the last passing threshold (warp 0's, lo, always passes)
                const unsigned pass = __ballot_sync(0xffffffffu, lane < kTreeWarps && sm.res[lane]);
                const int w = 31 - __clz(pass);
                if (lane == 0) {
                    sm.lo = sm.tw[w];
                    if (w + 1 < kTreeWarps) {
                        sm.hi = sm.tw[w + 1];
                        sm.hi_count = sm.cnt[w + 1];
                    }
                    sm.vfirst = 0;
                }
            }
            __syncthreads();
        }
    }
    if (!search) {
        if (threadIdx.x == 0) sm.lo = f2ord(0.f);
        __syncthreads();
    }
    const int take_all = search && sm.take_all;
    const uint32_t lo = sm.lo;
    const float tau = take_all ? -INFINITY : ord2f(lo);

    // 2. (warp 0) nodes strictly above tau, then materialise level by level
    //    in breadth-first order
    int n = 1;
    if (warp == 0) {
        int ties_left;
        if (take_all) {
            ties_left = budget;
        } else if (!search) {
            ties_left = 0;
        } else {
            // the search ended at hi = lo + 1, a tested threshold whose count
            // (below the budget, so exact) is the number of nodes above tau
            ties_left = budget - sm.hi_count;
        }
        if (lane == 0) {
            sm.nscore[0] = 0.f;
            sm.nparent[0] = -1;
            sm.nrank[0] = 0;
            sm.ndepth[0] = 0;
        }
        __syncwarp();
        int lvl_begin = 0, lvl_end = 1;
        for (int m = 0; m < D && lvl_begin < lvl_end && n < budget; ++m) {
            for (int c0 = lvl_begin; c0 < lvl_end; c0 += 32) {
                const int i = c0 + lane;
                const bool live = i < lvl_end;
                const float s = live ? sm.nscore[i] : 0.f;
                // a node's children above tau come first, then those equal to
                // it (the log-probs are sorted); per rank, one ballot each for
                // "above" and "equal" gives every lane its own counts and the
                // counts of the lanes before it (a prefix sum without a scan)
                const unsigned lt = (1u << lane) - 1u;
                int cgt = 0, ceq = 0, pre_gt = 0, pre_eq = 0, tot_gt = 0, tot_eq = 0;
                for (int r = 0; r < k; ++r) {
                    const float cs = __fadd_rn(s, sm.lp[m][r]);
                    const unsigned bg = __ballot_sync(0xffffffffu, live && cs > tau);
                    const unsigned be = __ballot_sync(0xffffffffu, live && cs == tau);
                    if ((bg | be) == 0u) break;
                    cgt += (bg >> lane) & 1u;
                    ceq += (be >> lane) & 1u;
                    pre_gt += __popc(bg & lt);
                    pre_eq += __popc(be & lt);
                    tot_gt += __popc(bg);
                    tot_eq += __popc(be);
                }
                // ties are taken in breadth-first order while the tie budget
                // lasts: the lanes before this one took min(pre_eq, ties_left)
                const int take_eq = max(0, min(ceq, ties_left - pre_eq));
                const int c = cgt + take_eq;
                const int used_eq = min(tot_eq, ties_left);
                const int tot = tot_gt + used_eq;
                const int off = n + pre_gt + min(pre_eq, ties_left);
                for (int r = 0; r < c && off + r < budget; ++r) {
                    sm.nscore[off + r] = __fadd_rn(s, sm.lp[m][r]);
                    sm.nparent[off + r] = i;
                    sm.nrank[off + r] = (uint8_t)r;
                    sm.ndepth[off + r] = (uint8_t)(m + 1);
                }
                n = min(budget, n + tot);
                ties_left -= used_eq;
            }
            __syncwarp();
            lvl_begin = lvl_end;
            lvl_end = n;
        }
        if (lane == 0) sm.nodes = n;              // node count for the other warps
    }
    __syncthreads();
    n = sm.nodes;

    // outputs; unused slots get parent -1, token -1, depth -1
    for (int i = threadIdx.x; i < budget; i += blockDim.x) {
        if (i < n) {
            const int d = sm.ndepth[i];
            o_par[i] = sm.nparent[i];
            o_dep[i] = d;
            const long long ti = (((long long)b * a.D) + (d - 1)) * k + sm.nrank[i];
            o_tok[i] = d == 0 ? a.root_token[b]
                       : (JSV_IN_BOUNDS(ti, (long long)a.B * a.D * k, a.status) ? a.topk_tokens[ti] : -1);
            if (o_sc) o_sc[i] = sm.nscore[i];
        } else {
            o_par[i] = -1;
            o_dep[i] = -1;
            o_tok[i] = -1;
            if (o_sc) o_sc[i] = -INFINITY;
        }
    }
    if (threadIdx.x == 0) a.num_nodes[b] = n;
}

cudaError_t launch_accum_logp_tree(const float *logp, const int32_t *topk_tokens, const int32_t *root_token, int B,
                                   int D, int k, int budget, int32_t *parent, int32_t *tokens, int32_t *depth,
                                   float *score, int32_t *num_nodes, int32_t *status, cudaStream_t st) {
    TreeArgs a{logp, topk_tokens, root_token, B, D, k, budget, parent, tokens, depth, score, num_nodes, status};
    const size_t smem = (size_t)kTreeWarps * 2 * kTreeLevel * sizeof(float);
    static PerDeviceOnce attr_once;
    cudaError_t ae = attr_once.run([&]() {
        cudaError_t e = cudaFuncSetAttribute(accum_logp_tree_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(accum_logp_tree_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        return e;
    });
    if (ae != cudaSuccess) return ae;
    cudaError_t e = launch_pdl(accum_logp_tree_kernel, dim3(B), dim3(32 * kTreeWarps), smem, st, a);
    count_launches(1);
    return e;
}

}  // namespace jsv
