/*
 * jsv.h -- C ABI of libjsv.so: the one-forward tree verification step of
 * causal parallel tree drafting (JetSpec), as hand-written CUDA for sm_100a.
 *
 * The method (JetSpec README, "JetSpec / Overview"): a draft head proposes a
 * token tree; the frozen target verifies the whole tree in ONE forward pass
 * under a tree-causal attention mask, and the accepted path is chosen by the
 * target's own logits, so decoding stays lossless.  The serving engine keeps
 * the KV cache in pages (README, "JetSpec / Quick Start": paged KV, custom
 * tree attention, CUDA graphs).  All reported runs are greedy (temperature 0).
 * One verify step is four calls on one stream, in this order:
 *
 *   jsv_tree_attention  tree-causal attention of every node over its
 *                       request's paged KV prefix plus its own ancestors
 *   jsv_lmhead_argmax   LM-head projection of every node's hidden state
 *                       fused with top-1 argmax (logits are never stored)
 *   jsv_accept_path     greedy longest-accepted-path walk
 *   jsv_kv_compact      move the accepted path's K/V rows to contiguous
 *                       slots P..P+a of each request (ragged batches)
 *
 * jsv_accept_compact does the last two in one launch.
 *
 * Conventions for every call
 *   - Pointers marked "device" are CUDA device (or managed) memory; the
 *     caller allocates and owns every buffer, workspace included.  The
 *     library never allocates, frees or synchronises.
 *   - bf16 tensors are IEEE bfloat16 bit patterns, row-major, contiguous.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are asynchronous: the return value covers host-side argument checks
 *     and the launch only.
 *   - Host-side checks return JSV_ERR_INVALID_ARG (NULL pointer, negative or
 *     inconsistent size, too-small workspace) or JSV_ERR_UNSUPPORTED (a
 *     shape outside the supported set) and launch nothing.
 *   - Errors that only the device can see (a malformed parent array, a page
 *     index outside [0, num_pages), node offsets that disagree with
 *     total_nodes, a path longer than max_path) are written to
 *     batch->dev_status (if non-NULL) with an atomic compare-and-swap from
 *     0, so the first error sticks; the affected request's work is skipped.
 *     Kernels never trap.  The caller zeroes *dev_status before a step.
 *   - Calls on distinct streams with distinct workspaces and outputs may run
 *     concurrently.
 */
#ifndef JSV_H
#define JSV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JSV_API __attribute__((visibility("default")))
#else
#define JSV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    JSV_OK = 0,
    JSV_ERR_INVALID_ARG = 1,   /* host-visible bad argument                  */
    JSV_ERR_UNSUPPORTED = 2,   /* shape outside the supported set            */
    JSV_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed       */
    JSV_ERR_TIMEOUT = 4,       /* a bounded device wait gave up              */
    JSV_ERR_DEVICE_INPUT = 5,  /* written to *dev_status: bad device data    */
    JSV_ERR_BOUNDS = 6         /* written to *dev_status, only by a library
                                  built with JSV_CHECK_BOUNDS: a computed
                                  index fell outside its buffer (a library
                                  fault; the access was skipped)            */
} jsv_status;

/*
 * Geometry of one verify step over B requests, shared by the calls that
 * touch the tree or the cache.
 *
 * Notation: request b has P_b committed prefix tokens and a draft tree of
 * N_b nodes (node 0 = root = the last committed token, whose K/V this
 * forward computes).  Nodes of all requests are packed: request b owns
 * global nodes node_offsets[b] .. node_offsets[b+1]-1, T = node_offsets[B].
 *
 * Tree: parent[] holds request-local indices with parent[0] = -1 and
 * 0 <= parent[i] < i for i > 0 (any topological order).
 *
 * Cache: k_cache and v_cache are [num_pages][page_size][Hkv][D] bf16.
 * Logical slot s of request b is row s % page_size of physical page
 * page_table[b * max_pages_per_req + s / page_size].  Slots [0, P_b) hold
 * the prefix; the caller has written tree node j's K/V at slot P_b + j, so
 * pages covering [0, P_b + N_b) must be mapped.
 */
typedef struct {
    int32_t B;                   /* requests, >= 1                                */
    int32_t Hq, Hkv, D;          /* query heads, KV heads (Hq % Hkv == 0), D in {64,128} */
    int32_t page_size;           /* must be 16                                    */
    int32_t max_pages_per_req;   /* row stride of page_table                      */
    int32_t num_pages;           /* physical pages in k_cache and in v_cache      */
    int32_t total_nodes;         /* T, must equal node_offsets[B]                 */
    int32_t max_nodes;           /* upper bound on N_b, 1..512                    */
    int32_t max_prefix;          /* upper bound on P_b, >= 0                      */
    const int32_t *page_table;   /* device [B][max_pages_per_req]                 */
    const int32_t *prefix_len;   /* device [B]   P_b                              */
    const int32_t *node_offsets; /* device [B+1]                                  */
    const int32_t *parent;       /* device [T]   request-local parent index       */
    int32_t *dev_status;         /* device [1] or NULL: first device-side error   */
} jsv_batch;

/* Bytes of scratch jsv_tree_attention needs for this geometry (split-KV
 * partial results; 0 when every request takes one split).  Depends on the
 * host-side fields and on the current device's SM count, which sets the
 * split count. */
JSV_API size_t jsv_tree_attention_workspace_size(const jsv_batch *batch);

/*
 * Tree-causal attention (README, "JetSpec / Overview": one forward pass under
 * a tree-causal mask).  For request b, node i, query head h, with
 * g = h / (Hq / Hkv), the visible sequence is prefix slots 0..P_b-1 followed
 * by slots P_b + j for every j on the root..i path (i included):
 *     out[t][h] = sum_j softmax_j(scale * <q[t][h], k_j>) * v_j
 * computed in fp32 from bf16 inputs and rounded to bf16.
 *   q        device [T][Hq][D] bf16, post-rotary
 *   k_cache, v_cache  device caches as described above (read only)
 *   scale    softmax scale (normally 1/sqrt(D))
 *   out      device [T][Hq][D] bf16
 *   workspace, workspace_bytes  device scratch of at least
 *            jsv_tree_attention_workspace_size(batch) bytes, 256-B aligned
 *            (NULL is accepted when that size is 0); any contents, since
 *            every call writes what it reads
 */
JSV_API jsv_status jsv_tree_attention(const jsv_batch *batch, const uint16_t *q,
                              const uint16_t *k_cache, const uint16_t *v_cache,
                              float scale, uint16_t *out,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * Budgeted draft-tree construction by cumulative log-probability (the pages'
 * default "accum_logp" tree: JetSpec README, "Evaluation", breadth-first and
 * kept by cumulative log-probability under depth, width and budget).  Reading:
 * for each request the draft head gives, per depth m = 1..depth, its top-width
 * candidate tokens with log-probabilities sorted in descending order.  A node
 * is a rank path; its score is the fp32 running sum of its edge log-probs
 * (added root to leaf).  The tree is the `budget` best nodes under
 *     score descending, depth ascending, rank path lexicographic ascending
 * (root = empty path, score 0, always kept), in breadth-first order with
 * children in rank order: parent[0] = -1 and parent[i] < i, ready for the
 * other calls.
 *   logp         device [B][depth][width] float, each row non-increasing, <= 0
 *   topk_tokens  device [B][depth][width] int32
 *   root_token   device [B] int32 (the last committed token)
 *   parent, tokens, node_depth  device [B][budget] int32 outputs; slots past
 *                num_nodes[b] get -1
 *   score        device [B][budget] float or NULL (fp32 node scores)
 *   num_nodes    device [B] int32: nodes emitted (budget, or fewer when the
 *                whole candidate tree is smaller)
 *   dev_status   device [1] int32 or NULL: a request whose log-probs are not
 *                sorted, positive or NaN gets JSV_ERR_DEVICE_INPUT and a
 *                root-only tree
 * Supported: 1 <= B, 0 <= depth <= 32, 1 <= width <= 32, 1 <= budget <= 512.
 */
JSV_API jsv_status jsv_accum_logp_tree(const float *logp, const int32_t *topk_tokens,
                                       const int32_t *root_token, int32_t B, int32_t depth,
                                       int32_t width, int32_t budget, int32_t *parent,
                                       int32_t *tokens, int32_t *node_depth, float *score,
                                       int32_t *num_nodes, int32_t *dev_status, void *stream);

/*
 * Tree Q/K/V projection with rotary positions, K/V appended to the paged cache
 * (the step before jsv_tree_attention; reading of the JetSpec README,
 * "JetSpec / Overview" and "Quick Start": one forward pass over the tree,
 * paged KV).  For node j of request b, qkv = w_qkv x_j with rows Q heads
 * (Hq*D), then K heads (Hkv*D), then V heads (Hkv*D); Q and K heads are
 * rotated at position P_b + depth(j) with the rotate-half pairs (i, i + D/2):
 *     out_i = x_i c_i - x_{i+D/2} s_i,  out_{i+D/2} = x_{i+D/2} c_i + x_i s_i
 * Q is written to q[j], K and V to logical slot P_b + j of the request's
 * pages.  fp32 accumulation, bf16 outputs.
 *   x          device [T][d] bf16 (the tree's hidden states entering the layer)
 *   w_qkv      device [(Hq + 2 Hkv) D][d] bf16
 *   rope_cos, rope_sin  device [max_pos][D/2] float tables
 *   q          device [T][Hq][D] bf16 output
 *   k_cache, v_cache  the paged caches; only tree slots P_b .. P_b+N_b-1 change
 * A node whose position reaches max_pos, or whose parent chain or page is
 * malformed, is skipped and JSV_ERR_DEVICE_INPUT is written to dev_status.
 * Supported: d % 64 == 0, 64 <= d <= 16384.
 */
JSV_API jsv_status jsv_tree_qkv_rope(const jsv_batch *batch, const uint16_t *x, const uint16_t *w_qkv,
                                     int32_t d, const float *rope_cos, const float *rope_sin,
                                     int32_t max_pos, uint16_t *q, uint16_t *k_cache,
                                     uint16_t *v_cache, void *stream);

/* Bytes of scratch jsv_lmhead_argmax needs (one 64-bit key per node and a
 * completion counter). */
JSV_API size_t jsv_lmhead_argmax_workspace_size(int32_t T, int32_t d, int32_t V);

/*
 * LM head fused with top-1 argmax (README, "JetSpec / Overview": the path is
 * selected by the target's own logits; temperature 0).
 *     argmax[t] = smallest v attaining max_v sum_k hidden[t][k] * w[v][k]
 * accumulated in fp32 from bf16; logits are never written to memory.
 *   hidden     device [T][d] bf16
 *   w          device [V][d] bf16 (the LM-head weight, row per token)
 *   argmax     device [T] int32
 *   max_logit  device [T] float (the fp32 maximum) or NULL
 *   workspace  device scratch of jsv_lmhead_argmax_workspace_size() bytes,
 *              8-B aligned, ZERO-FILLED before its first use (e.g. one
 *              cudaMemsetAsync when it is allocated); every call leaves it
 *              zero-filled again, so it is reused without clearing.
 *   dev_status device [1] int32 or NULL.  A bounded wait of the kernel that
 *              gave up writes JSV_ERR_TIMEOUT (compare-and-swap from 0); the
 *              call's argmax and max_logit are then unspecified, and the
 *              workspace is still left zero-filled (every CTA counts the work
 *              it took, finished or abandoned, and the CTA that completes the
 *              count clears the keys and the counter).
 * Ordering: the kernel reads `hidden` and `w` while the previous launch on
 * the stream may still be running (it waits for that launch only before it
 * touches the workspace and the outputs), so the tree-attention kernels of
 * the same step run beside its main loop.  Kernels of other libraries are
 * complete before it starts, as usual; only a buffer written by an earlier
 * call of THIS library that may still be in flight (for instance
 * jsv_tree_attention's `out`) must not be passed as `hidden` or `w`.
 * Supported: 1 <= T, d % 64 == 0, 64 <= d <= 16384, 1 <= V < 2^31.
 */
JSV_API jsv_status jsv_lmhead_argmax(const uint16_t *hidden, const uint16_t *w,
                             int32_t T, int32_t d, int32_t V,
                             int32_t *argmax, float *max_logit,
                             void *workspace, size_t workspace_bytes,
                             int32_t *dev_status, void *stream);

/*
 * Greedy accept walk (README, "JetSpec / Overview": lossless by
 * construction; "tokens per forward" = accepted + 1).  Per request, start at
 * the root (always accepted); while some child c of the current node has
 * tokens[c] == argmax[current], move to the smallest such c.
 *   tokens      device [T] int32, the draft token of every node
 *   argmax      device [T] int32, the target's choice at every node
 *   max_path    row length of `path` (>= 1)
 *   path        device [B][max_path] int32: request-local indices of the
 *               accepted path starting with 0, then -1 padding
 *   accept_len  device [B] int32: accepted draft nodes a = path length - 1
 *   bonus       device [B] int32: argmax at the last accepted node
 * A path that would exceed max_path sets JSV_ERR_DEVICE_INPUT and is cut.
 */
JSV_API jsv_status jsv_accept_path(const jsv_batch *batch, const int32_t *tokens,
                           const int32_t *argmax, int32_t max_path,
                           int32_t *path, int32_t *accept_len, int32_t *bonus,
                           void *stream);

/*
 * Accepted-path KV compaction (README, "JetSpec / Quick Start": paged KV).
 * For every request and k = 0..a: the K and V rows (all KV heads) of slot
 * P_b + path[k] move to slot P_b + k, with the result of an in-order copy
 * (every source is read before any destination is written).  Slots other
 * than P_b..P_b+a are untouched.  new_len[b] = P_b + a + 1.
 *   k_cache, v_cache  device caches, updated in place
 *   path, accept_len  as written by jsv_accept_path (max_path = row stride)
 *   new_len           device [B] int32
 */
JSV_API jsv_status jsv_kv_compact(const jsv_batch *batch, uint16_t *k_cache, uint16_t *v_cache,
                          const int32_t *path, int32_t max_path, const int32_t *accept_len,
                          int32_t *new_len, void *stream);

/*
 * jsv_accept_path followed by jsv_kv_compact, in one kernel launch: the
 * step's two latency-bound tail calls fused (the pages have no counterpart;
 * a deployment form of the same two operations).  Every output -- path,
 * accept_len, bonus, the K/V caches and new_len -- and every device-side
 * error equals what the two calls in sequence produce on the same inputs.
 * Arguments follow those two calls: the tree arrays and argmax are read, the
 * path row is written with stride max_path, and the caches are updated in
 * place.  Every argument, the batch geometry included, is read only after
 * the previous launch on the stream has completed, so new_len of one step
 * may be passed back as the next step's prefix_len.
 */
JSV_API jsv_status jsv_accept_compact(const jsv_batch *batch, const int32_t *tokens,
                                      const int32_t *argmax, int32_t max_path,
                                      int32_t *path, int32_t *accept_len, int32_t *bonus,
                                      uint16_t *k_cache, uint16_t *v_cache, int32_t *new_len,
                                      void *stream);

/*
 * LM head fused with top-1 argmax for callers that cannot allocate device
 * memory (a region under CUDA-graph capture, a plugin whose host owns every
 * allocation, a loop that cannot afford cudaMalloc's synchronisation).
 * The pages have no counterpart: it is a deployment variant of
 * jsv_lmhead_argmax with the same result, whose scratch (one 64-bit key per
 * node) is a fixed file-scope device array inside the library instead of a
 * workspace argument.  The caller still passes inputs and outputs.
 *   - T must be <= JSV_NOALLOC_MAX_NODES, else JSV_ERR_UNSUPPORTED; the
 *     other arguments, dev_status included, follow jsv_lmhead_argmax.
 *   - The array ((JSV_NOALLOC_MAX_NODES + 1) * 8 bytes) is held on every GPU
 *     that loads the library until the process exits.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.
 *   - Nothing is allocated or freed: no cudaMalloc, cudaFree or allocating
 *     library routine.  The array starts zeroed and every call leaves the
 *     keys it used and the counter zeroed again, a call that reported
 *     JSV_ERR_TIMEOUT included (its outputs are then unspecified).
 *   - Every call shares the one array, which keeps the last call's contents:
 *     calls whose kernels overlap on the GPU (different streams, or
 *     different host threads on one device) race and give wrong results.
 *     Serialise them on one stream.
 */
#define JSV_NOALLOC_MAX_NODES 8192
JSV_API jsv_status jsv_lmhead_argmax_noalloc(const uint16_t *hidden, const uint16_t *w,
                                             int32_t T, int32_t d, int32_t V,
                                             int32_t *argmax, float *max_logit,
                                             int32_t *dev_status, void *stream);

/* Number of kernels this library has launched in the calling process since
 * it was loaded (all devices, all streams).  A diagnostic for counting the
 * launches inside a timed region; not tied to any stream order. */
JSV_API uint64_t jsv_kernel_launches(void);

/*
 * Failure-detection self-test of the bounded device waits.  Every wait of
 * the library's tensor-core kernels on an mbarrier gives up after a time
 * limit, writes JSV_ERR_TIMEOUT to the status word and unwinds (copies in
 * flight drained, TMEM released), so a lost arrival ends in a readable status
 * rather than a hung GPU.  This call launches one CTA that waits on a barrier
 * nothing signals, with the limit shortened to `limit_us` microseconds
 * (1 .. 2,000,000); it writes JSV_ERR_TIMEOUT to *dev_status (device int32,
 * compare-and-swap from 0) and exits, leaving the context usable.
 */
JSV_API jsv_status jsv_selftest_wait_timeout(int32_t *dev_status, uint32_t limit_us, void *stream);

/*
 * Failure-detection self-test of the LM head's timeout path.  Runs the LM head
 * exactly as jsv_lmhead_argmax does with `workspace` (or, with workspace
 * NULL, as jsv_lmhead_argmax_noalloc does, on the library's scratch array),
 * except that the producer warp of the first CTA -- the first CTA pair for
 * trees above 128 nodes -- first waits on a barrier that nothing signals,
 * with the limit shortened to `limit_us` microseconds (1 .. 2,000,000).  That
 * wait gives up before the CTA has issued any copy: the CTA writes
 * JSV_ERR_TIMEOUT to *dev_status (device int32, required, compare-and-swap
 * from 0), stops, and the rest of the grid completes.  argmax and max_logit
 * are then unspecified; the workspace (or scratch array) is left zeroed, so
 * the next ordinary call on it returns the right result.  Other arguments
 * and checks follow jsv_lmhead_argmax (and the T limit of the no-alloc form).
 */
JSV_API jsv_status jsv_selftest_lmhead_timeout(const uint16_t *hidden, const uint16_t *w,
                                               int32_t T, int32_t d, int32_t V,
                                               int32_t *argmax, float *max_logit,
                                               void *workspace, size_t workspace_bytes,
                                               int32_t *dev_status, uint32_t limit_us, void *stream);

/* Text of the last CUDA error behind a JSV_ERR_CUDA returned to the calling
 * host thread (a launch or runtime call that failed), or a fixed message if
 * none was recorded; for a failed kernel launch it also names the kernel's
 * registers and shared memory against the launch.  The string belongs to the
 * calling thread and stays valid until its next call; later successful calls
 * do not clear it. */
JSV_API const char *jsv_last_error_string(void);

/* Static string for a status code. */
JSV_API const char *jsv_status_string(jsv_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
JSV_API int32_t jsv_version(void);

/* Build flags of this library: bit 0 set when it was compiled with
 * JSV_CHECK_BOUNDS (libjsv_checked.so), i.e. every computed global index
 * of the kernels is compared with its buffer's extent before the access and
 * a miss is skipped and written to the status word as JSV_ERR_BOUNDS.  The
 * pages have no counterpart: it is a debugging aid of this library. */
JSV_API int32_t jsv_build_flags(void);

#ifdef __cplusplus
}
#endif

#endif /* JSV_H */
