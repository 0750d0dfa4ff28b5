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
// One warp per request, no sorting and no heap:
//  1. tau, the budget-th best score, by binary search over the fp32 order:
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

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

struct TreeSmem {
    float lp[kTreeMaxDepth][kTreeMaxWidth];
    float lvl[2][kTreeMaxBudget + kTreeMaxWidth];
    float nscore[kTreeMaxBudget];
    int32_t nparent[kTreeMaxBudget];
    uint8_t nrank[kTreeMaxBudget];
    uint8_t ndepth[kTreeMaxBudget];
};

// Number of nodes with score >= x, capped at `cap` (exits as soon as it is
// reached).  Warp-cooperative; the result is uniform.
__device__ int count_ge(TreeSmem &sm, int D, int k, float x, int cap, int lane) {
    float *cur = sm.lvl[0], *nxt = sm.lvl[1];
    if (lane == 0) cur[0] = 0.f;
    __syncwarp();
    int ncur = 1, total = 1;
    if (total >= cap) return cap;
    for (int m = 0; m < D && ncur > 0; ++m) {
        int base = 0;
        for (int c0 = 0; c0 < ncur; c0 += 32) {
            const int i = c0 + lane;
            float s = 0.f;
            int cnt = 0;
            if (i < ncur) {
                s = cur[i];
                for (int r = 0; r < k; ++r) {
                    if (__fadd_rn(s, sm.lp[m][r]) >= x) ++cnt;
                    else break;
                }
            }
            const int incl = warp_incl_scan(cnt, lane);
            const int tot = __shfl_sync(0xffffffffu, incl, 31);
            if (total + base + tot >= cap) return cap;
            const int off = base + incl - cnt;
            for (int r = 0; r < cnt; ++r) nxt[off + r] = __fadd_rn(s, sm.lp[m][r]);
            base += tot;
        }
        __syncwarp();
        total += base;
        ncur = base;
        float *t = cur; cur = nxt; nxt = t;
    }
    return total;
}

__global__ void __launch_bounds__(32)
accum_logp_tree_kernel(TreeArgs a) {
    pdl_allow_dependents();
    pdl_wait_predecessor();
    __shared__ TreeSmem sm;
    const int b = blockIdx.x, lane = threadIdx.x;
    int D = a.D;
    const int k = a.k, budget = a.budget;
    int32_t *o_par = a.parent + (size_t)b * budget;
    int32_t *o_tok = a.tokens + (size_t)b * budget;
    int32_t *o_dep = a.depth + (size_t)b * budget;
    float *o_sc = a.score ? a.score + (size_t)b * budget : nullptr;

    // stage and validate the log-probs: finite or -inf, <= 0, non-increasing per depth
    bool bad = false;
    for (int e = lane; e < D * k; e += 32) {
        const float v = a.logp[((size_t)b * D) * k + e];
        const int r = e % k;
        bad |= !(v <= 0.f) && !(v == -INFINITY);
        sm.lp[e / k][r] = v;
    }
    __syncwarp();
    for (int e = lane; e < D * k; e += 32) {
        const int m = e / k, r = e % k;
        if (r > 0 && !(sm.lp[m][r] <= sm.lp[m][r - 1])) bad = true;
    }
    if (__any_sync(0xffffffffu, bad)) {
        if (lane == 0) flag_error(a.status, JSV_ERR_DEVICE_INPUT);
        D = 0;    // emit the root alone
    }

    // 1. tau: the largest x with count(x) >= budget, by bisection over the fp32 order
    int take_all = 0;
    uint32_t lo = f2ord(-INFINITY), hi = f2ord(0.f) + 1u;
    if (budget <= 1 || D == 0) {
        take_all = 0;
        lo = f2ord(0.f);
    } else if (count_ge(sm, D, k, -INFINITY, budget, lane) < budget) {
        take_all = 1;                     // the whole candidate tree fits the budget
    } else {
        while (hi - lo > 1u) {
            const uint32_t mid = lo + (hi - lo) / 2u;
            if (count_ge(sm, D, k, ord2f(mid), budget, lane) >= budget) lo = mid;
            else hi = mid;
        }
    }
    const float tau = take_all ? -INFINITY : ord2f(lo);
    // nodes strictly above tau (uncapped count is < budget by the bisection)
    int ties_left;
    if (take_all) {
        ties_left = budget;
    } else if (budget <= 1 || D == 0) {
        ties_left = 0;
    } else {
        const int n_gt = lo == f2ord(0.f) ? count_ge(sm, D, k, __uint_as_float(0x00000001u), budget, lane)
                                          : count_ge(sm, D, k, ord2f(lo + 1u), budget, lane);
        ties_left = budget - n_gt;
    }

    // 2. materialise level by level in breadth-first order
    if (lane == 0) {
        sm.nscore[0] = 0.f;
        sm.nparent[0] = -1;
        sm.nrank[0] = 0;
        sm.ndepth[0] = 0;
    }
    __syncwarp();
    int n = 1, lvl_begin = 0, lvl_end = 1;
    for (int m = 0; m < D && lvl_begin < lvl_end && n < budget; ++m) {
        for (int c0 = lvl_begin; c0 < lvl_end; c0 += 32) {
            const int i = c0 + lane;
            float s = 0.f;
            int cgt = 0, ceq = 0;
            if (i < lvl_end) {
                s = sm.nscore[i];
                for (int r = 0; r < k; ++r) {
                    const float cs = __fadd_rn(s, sm.lp[m][r]);
                    if (cs > tau) ++cgt;
                    else if (cs == tau) ++ceq;
                    else break;
                }
            }
            // ties are taken in breadth-first order while the tie budget lasts
            const int eq_incl = warp_incl_scan(ceq, lane);
            const int eq_excl = eq_incl - ceq;
            const int take_eq = max(0, min(ceq, ties_left - eq_excl));
            const int c = cgt + take_eq;
            const int incl = warp_incl_scan(c, lane);
            const int tot = __shfl_sync(0xffffffffu, incl, 31);
            const int used_eq = __shfl_sync(0xffffffffu, max(0, min(eq_incl, ties_left)), 31);
            const int off = n + incl - c;
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

    // outputs; unused slots get parent -1, token -1, depth -1
    for (int i = lane; i < budget; i += 32) {
        if (i < n) {
            const int d = sm.ndepth[i];
            o_par[i] = sm.nparent[i];
            o_dep[i] = d;
            o_tok[i] = d == 0 ? a.root_token[b]
                              : a.topk_tokens[(((size_t)b * a.D) + (d - 1)) * k + sm.nrank[i]];
            if (o_sc) o_sc[i] = sm.nscore[i];
        } else {
            o_par[i] = -1;
            o_dep[i] = -1;
            o_tok[i] = -1;
            if (o_sc) o_sc[i] = -INFINITY;
        }
    }
    if (lane == 0) a.num_nodes[b] = n;
}

cudaError_t launch_accum_logp_tree(const float *logp, const int32_t *topk_tokens, const int32_t *root_token, int B,
                                   int D, int k, int budget, int32_t *parent, int32_t *tokens, int32_t *depth,
                                   float *score, int32_t *num_nodes, int32_t *status, cudaStream_t st) {
    TreeArgs a{logp, topk_tokens, root_token, B, D, k, budget, parent, tokens, depth, score, num_nodes, status};
    cudaError_t e = launch_pdl(accum_logp_tree_kernel, dim3(B), dim3(32), 0, st, a);
    count_launches(1);
    return e;
}

}  // namespace jsv
