// Greedy accept walk of one request by one warp, over the request's parent,
// draft-token and target-argmax arrays staged in shared memory.  Shared by
// jsv_accept_path and jsv_accept_compact.
//
// JetSpec README, "JetSpec / Overview": the accepted path is chosen by the
// target's own logits, so decoding is lossless.  At temperature 0 that is
// the greedy descent: from the root, step to the smallest-index child whose
// draft token equals the target's argmax at the current node, until no
// child matches.  One pass over the nodes, a node per lane, records for
// every node the smallest index of a child whose draft token equals the
// node's argmax (a shared-memory atomicMin); the walk then follows these
// links from the root, one shared-memory load per accepted token.
#pragma once

#include "jsv_internal.cuh"

namespace jsv {

constexpr int kWalkMaxNodes = 512;

// Walks the tree of n nodes (parents already checked: 0 <= parent[j] < j
// for j > 0); lane 0 writes path entries 1, 2, ... to `out` (entry 0 is the
// root and is the caller's).  `s_next` is [n] shared scratch.  Returns the
// path length, root included; `last` receives the last accepted node and
// `cut` is set when a further match would make the path longer than
// max_path (the walk stops there).  Every lane of the warp must call it.
__device__ __forceinline__ int greedy_walk_warp(const int32_t *s_par, const int32_t *s_tok, const int32_t *s_arg,
                                                int32_t *s_next, int n, int max_path, int32_t *out, int lane,
                                                int &last, bool &cut) {
    for (int j = lane; j < n; j += 32) s_next[j] = n;          // no accepted child
    __syncwarp();
    for (int j = 1 + lane; j < n; j += 32) {
        const int p = s_par[j];
        if (s_tok[j] == s_arg[p]) atomicMin(&s_next[p], j);
    }
    __syncwarp();
    int cur = 0, len = 1;
    cut = false;
    while (true) {
        const int nx = s_next[cur];
        if (nx >= n) break;
        if (len >= max_path) {
            cut = true;
            break;
        }
        if (lane == 0) out[len] = nx;
        ++len;
        cur = nx;
    }
    last = cur;
    return len;
}

}  // namespace jsv
