// Greedy accept walk of one request by one warp, over the request's parent,
// draft-token and target-argmax arrays staged in shared memory.  Shared by
// jsv_accept_path and jsv_accept_compact.
//
// JetSpec README, "JetSpec / Overview": the accepted path is chosen by the
// target's own logits, so decoding is lossless.  At temperature 0 that is
// the greedy descent: from the root, step to the smallest-index child whose
// draft token equals the target's argmax at the current node, until no
// child matches.  Children have larger indices than their parent
// (topological order), so each step scans indices > cur with a warp ballot
// and takes the lowest set lane of the first chunk that has a match.
#pragma once

#include "jsv_internal.cuh"

namespace jsv {

constexpr int kWalkMaxNodes = 512;

// Walks the tree of n nodes; lane 0 writes path entries 1, 2, ... to `out`
// (entry 0 is the root and is the caller's).  Returns the path length, root
// included; `last` receives the last accepted node and `cut` is set when a
// further match would make the path longer than max_path (the walk stops
// there).  Every lane of the warp must call it.
__device__ __forceinline__ int greedy_walk_warp(const int32_t *s_par, const int32_t *s_tok, const int32_t *s_arg,
                                                int n, int max_path, int32_t *out, int lane, int &last, bool &cut) {
    int cur = 0, len = 1;
    cut = false;
    while (true) {
        const int want = s_arg[cur];
        int found = -1;
        for (int j0 = cur + 1; j0 < n; j0 += 32) {
            const int j = j0 + lane;
            const bool m = j < n && s_par[j] == cur && s_tok[j] == want;
            const unsigned bal = __ballot_sync(0xffffffffu, m);
            if (bal) { found = j0 + __ffs(bal) - 1; break; }
        }
        if (found < 0) break;
        if (len >= max_path) {
            cut = true;
            break;
        }
        if (lane == 0) out[len] = found;
        ++len;
        cur = found;
    }
    last = cur;
    return len;
}

}  // namespace jsv
