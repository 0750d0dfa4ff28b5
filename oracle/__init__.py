"""Oracle for the one-forward tree verification step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import or run anything here.  The
product library never calls it, and the oracle shares no code with the CUDA
path: the two meet only at the seeded input generator, which holds none of
the method's arithmetic.

What it computes, each part written from the JetSpec README ("JetSpec /
Overview": a draft token tree is verified in one forward pass of the frozen
target under a tree-causal attention mask, and the accepted path is chosen by
the target's own logits, so decoding stays lossless; all reported runs use
temperature 0):

* ``tree_attention``   plain fp64 attention of every (node, head) row over
                       the prefix plus the node's root-to-node path
                       (``tree_attention.c``).
* ``lmhead_top2``      fp64 logits H @ W^T (a library matmul as the step),
                       the smallest index attaining the maximum, and the
                       runner-up value.
* ``certify_margin``   whether the top-1 choice is decided the same way by
                       any fp32 summation order (a reading of the lossless
                       greedy rule for a kernel that accumulates in fp32).
* ``accept_path``      the greedy walk: from the root, repeatedly descend to
                       the smallest-index child whose token equals the
                       target's argmax at the current node.
* ``kv_compact``       copy the accepted path's K/V rows to slots P..P+a in
                       increasing order; new length P+a+1.

Every function is pinned in ``tests/test_oracle_*.py`` against brute force,
closed forms, invariants or library routines.  The end-to-end throughput the
pages report is not reproducible here (no weights or datasets): parity
unpinned for that quantity only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SO = _HERE / "_tree_attention.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile the C part of the oracle with the host compiler."""
    src = _HERE / "tree_attention.c"
    if force or not _SO.exists() or _SO.stat().st_mtime < src.stat().st_mtime:
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               str(src), "-o", str(_SO), "-lm"])
    return _SO


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_SO))
        p = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_tree_attention.argtypes = [i, i, i, i, i, i, p, p, p, p, p, p, p,
                                              ctypes.c_double, p, i, p, i]
        lib.oracle_tree_attention.restype = i
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Tree attention
# ---------------------------------------------------------------------------

def tree_attention(*, Hq, Hkv, D, page_table, prefix_len, node_offsets, parent,
                   q, k_cache, v_cache, scale, rows=None, page_size=16, threads=None):
    """fp64 outputs for the requested (global node, head) rows.

    ``rows`` is an int array [n, 2]; None means every row, returned as
    [T, Hq, D].  Inputs are bf16 bit patterns (uint16)."""
    lib = _load()
    page_table = np.ascontiguousarray(page_table, dtype=np.int32)
    prefix_len = np.ascontiguousarray(prefix_len, dtype=np.int32)
    node_offsets = np.ascontiguousarray(node_offsets, dtype=np.int32)
    parent = np.ascontiguousarray(parent, dtype=np.int32)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.uint16)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.uint16)
    T = int(node_offsets[-1])
    full = rows is None
    if full:
        tt, hh = np.meshgrid(np.arange(T), np.arange(Hq), indexing="ij")
        rows = np.stack([tt.ravel(), hh.ravel()], axis=1)
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    out = np.zeros((len(rows), D), dtype=np.float64)
    B = len(prefix_len)
    st = lib.oracle_tree_attention(B, Hq, Hkv, D, page_size, page_table.shape[1],
                                   _ptr(page_table), _ptr(prefix_len), _ptr(node_offsets),
                                   _ptr(parent), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                   float(scale), _ptr(rows), len(rows), _ptr(out),
                                   threads or host_threads())
    if st != 0:
        raise ValueError("oracle_tree_attention: malformed tree or row list")
    return out.reshape(T, Hq, D) if full else out


def tree_attention_wl(wl, rows=None, threads=None):
    return tree_attention(Hq=wl.Hq, Hkv=wl.Hkv, D=wl.D, page_table=wl.page_table,
                          prefix_len=wl.prefix_len, node_offsets=wl.node_offsets,
                          parent=wl.parent, q=wl.q, k_cache=wl.k_cache, v_cache=wl.v_cache,
                          scale=wl.scale, rows=rows, threads=threads)


# ---------------------------------------------------------------------------
# LM head + argmax
# ---------------------------------------------------------------------------

def lmhead_top2(hidden, w, rows=None, chunk=8192):
    """fp64 logits l[i, v] = sum_k H[i,k] W[v,k] for the given rows; returns
    (argmax, top1 value, runner-up value).  argmax is the smallest v that
    attains the maximum (temperature-0 greedy choice).  The matmul is the
    library step; vocabulary chunks are visited in increasing order and a
    later chunk replaces the running best only on a strictly larger value."""
    H = bf16_to_f64(hidden if rows is None else np.asarray(hidden)[rows])
    T = H.shape[0]
    V = w.shape[0]
    best = np.full(T, -np.inf)
    second = np.full(T, -np.inf)
    arg = np.zeros(T, dtype=np.int64)
    r = np.arange(T)
    for v0 in range(0, V, chunk):
        Wc = bf16_to_f64(w[v0:v0 + chunk])
        L = H @ Wc.T
        j = np.argmax(L, axis=1)
        top = L[r, j]
        L[r, j] = -np.inf
        nxt = L.max(axis=1) if L.shape[1] > 1 else np.full(T, -np.inf)
        upd = top > best
        # runner-up over everything seen so far
        second = np.where(upd, np.maximum(best, nxt), np.maximum(second, top))
        best = np.where(upd, top, best)
        arg = np.where(upd, v0 + j, arg)
    return arg, best, second


def lmhead_argmax(hidden, w, rows=None):
    a, _, _ = lmhead_top2(hidden, w, rows)
    return a


def w_row_norm_max(w):
    """max_v |W_v|_2 in fp64."""
    m = 0.0
    for v0 in range(0, w.shape[0], 16384):
        Wc = bf16_to_f64(w[v0:v0 + 16384])
        m = max(m, float(np.sqrt((Wc * Wc).sum(axis=1)).max()))
    return m


def certify_margin(hidden, w, argmax, top1, top2, rows=None, safety=4.0, wmax=None):
    """Per row: is the top-1 choice the same under every fp32 summation order?

    A kernel that forms each logit as an fp32 sum of the d exact bf16*bf16
    products is within gamma * sum_k |H_k W_vk| of the exact value, with
    gamma = d * 2^-24 for round-to-nearest (the standard recursive-summation
    bound); ``safety`` widens it for accumulators that truncate or align
    products before adding.  For v != v1, sum_k |H_k W_vk| <= |H|_2 |W_v|_2
    (Cauchy-Schwarz).  So the choice is certain when
        l1 - l2 > safety * gamma * (A_v1 + |H|_2 * max_v |W_v|_2).
    Returns (certified bool [n], margin/bound ratio [n])."""
    H = bf16_to_f64(hidden if rows is None else np.asarray(hidden)[rows])
    d = H.shape[1]
    Wmax = w_row_norm_max(w) if wmax is None else wmax
    W1 = bf16_to_f64(w[np.asarray(argmax, dtype=np.int64)])
    A1 = np.abs(H * W1).sum(axis=1)
    hn = np.sqrt((H * H).sum(axis=1))
    bound = safety * d * 2.0 ** -24 * (A1 + hn * Wmax)
    gap = np.asarray(top1) - np.asarray(top2)
    return gap > bound, gap / bound


# ---------------------------------------------------------------------------
# Greedy accept walk and KV compaction
# ---------------------------------------------------------------------------

def accept_path(parent, tokens, argmax):
    """One request, request-local indices.  Start at the root (always
    accepted).  While some child c of the current node carries the token the
    target chooses at the current node, move to the smallest such c.
    Returns (path as local indices starting with 0, accept_len, bonus token),
    accept_len = number of accepted draft nodes = len(path) - 1, and the
    bonus is the target's choice at the last accepted node."""
    n = len(parent)
    cur = 0
    path = [0]
    while True:
        want = int(argmax[cur])
        nxt = None
        for c in range(n):
            if int(parent[c]) == cur and int(tokens[c]) == want:
                nxt = c
                break
        if nxt is None:
            break
        path.append(nxt)
        cur = nxt
    return path, len(path) - 1, int(argmax[cur])


def accept_batch(node_offsets, parent, tokens, argmax):
    out = []
    for b in range(len(node_offsets) - 1):
        s, e = int(node_offsets[b]), int(node_offsets[b + 1])
        out.append(accept_path(parent[s:e], tokens[s:e], argmax[s:e]))
    return out


def kv_compact(k_cache, v_cache, page_table, prefix_len, paths, page_size=16):
    """In place: for every request, for k = 0..a in increasing order, copy
    the K and V rows (all KV heads) of logical slot P + path[k] to logical
    slot P + k.  Returns new lengths P + a + 1.  Because path[k] >= k, the
    increasing order never reads a slot it has already overwritten."""
    new_len = []
    for b, path in enumerate(paths):
        P = int(prefix_len[b])
        for k, src_node in enumerate(path):
            src = P + int(src_node)
            dst = P + k
            sp, so = int(page_table[b, src // page_size]), src % page_size
            dp, do = int(page_table[b, dst // page_size]), dst % page_size
            k_cache[dp, do] = k_cache[sp, so]
            v_cache[dp, do] = v_cache[sp, so]
        new_len.append(P + len(path))
    return np.asarray(new_len, dtype=np.int32)


# ---------------------------------------------------------------------------
# Budgeted tree construction by cumulative log-probability (accum_logp)
# ---------------------------------------------------------------------------

def accum_logp_tree(logp, topk_tokens, root_token, budget):
    """The draft tree the pages' default ``accum_logp`` construction keeps
    (JetSpec README, "Evaluation": a breadth-first tree kept by cumulative
    log-probability under depth, width and budget).

    Reading: the draft head gives, for each depth m = 1..D, its top-k
    candidate tokens with log-probabilities sorted in descending order
    (``logp[m-1][r]``, ``topk_tokens[m-1][r]``).  A node is a rank path
    (r_1..r_m); its score is the fp32 running sum of its edge log-probs, added
    root-to-leaf (the kernel's precision decides the comparison).  The tree
    is the ``budget`` best nodes under the total order
        score descending, then depth ascending, then the rank path read as a
        base-k number ascending,
    the root (empty path, score 0) included.  Children never outrank their
    parent and a rank never outranks the previous rank, so that set is
    ancestor- and sibling-closed.  It is returned in breadth-first order
    (level by level, children by parent order then rank).

    Best-first expansion visits nodes in exactly that order: a node enters
    the candidate set when its parent (first child) or its previous sibling
    is taken.  Returns dict(parent, tokens, depth, score, code) as numpy
    arrays of length n <= budget."""
    import heapq
    logp = np.asarray(logp, dtype=np.float32)
    topk_tokens = np.asarray(topk_tokens)
    D, k = logp.shape
    sel = [(-1, -1, 0, np.float32(0.0), 0)]        # (parent sel index, rank, depth, score, code)
    heap = []

    def push(parent_sel, rank, depth):
        ps = sel[parent_sel][3]
        s = np.float32(ps + logp[depth - 1][rank])
        code = sel[parent_sel][4] * k + rank
        heapq.heappush(heap, (-float(s), depth, code, parent_sel, rank, s))

    if D >= 1 and k >= 1 and budget > 1:
        push(0, 0, 1)
    while heap and len(sel) < budget:
        _, depth, code, parent_sel, rank, s = heapq.heappop(heap)
        me = len(sel)
        sel.append((parent_sel, rank, depth, s, code))
        if rank + 1 < k:
            push(parent_sel, rank + 1, depth)
        if depth < D:
            push(me, 0, depth + 1)
    # breadth-first relabelling
    n = len(sel)
    kids = [[] for _ in range(n)]
    for i in range(1, n):
        kids[sel[i][0]].append(i)
    for c in kids:
        c.sort(key=lambda i: sel[i][1])
    order = [0]
    head = 0
    while head < len(order):
        order.extend(kids[order[head]])
        head += 1
    new = {old: new_i for new_i, old in enumerate(order)}
    parent = np.array([-1] + [new[sel[o][0]] for o in order[1:]], dtype=np.int32)
    depth = np.array([sel[o][2] for o in order], dtype=np.int32)
    tokens = np.array([int(root_token)] + [int(topk_tokens[sel[o][2] - 1][sel[o][1]]) for o in order[1:]],
                      dtype=np.int32)
    score = np.array([sel[o][3] for o in order], dtype=np.float32)
    code = np.array([sel[o][4] for o in order], dtype=np.uint64)
    return dict(parent=parent, tokens=tokens, depth=depth, score=score, code=code)


# ---------------------------------------------------------------------------
# Tree Q/K/V projection with rotary positions, K/V appended to the paged cache
# ---------------------------------------------------------------------------

def rope_rotate(x, cos, sin):
    """Rotate-half rotary embedding of one head vector x (length D) with the
    pair tables cos/sin (length D/2): out_i = x_i c_i - x_{i+D/2} s_i and
    out_{i+D/2} = x_{i+D/2} c_i + x_i s_i."""
    h = len(x) // 2
    a, b = x[:h], x[h:]
    return np.concatenate([a * cos - b * sin, b * cos + a * sin])


def tree_qkv_rope(*, x, w_qkv, Hq, Hkv, D, page_table, prefix_len, node_offsets, parent,
                  rope_cos, rope_sin, k_cache, v_cache, page_size=16):
    """The step on the other side of the tree attention (reading of the JetSpec
    README, "JetSpec / Overview" and "Quick Start": one forward over the tree
    with a paged KV cache).  For node j of request b: qkv = W_qkv x_j (fp64;
    rows Q heads, then K heads, then V heads); Q and K heads are rotated at
    position P_b + depth(j) (a node sits one position after its parent); K and
    V heads are written to logical slot P_b + j of the request's pages.
    Returns q as float64 [T][Hq][D]; k_cache/v_cache (uint16 bf16 bits) are
    updated in place with the fp64 K/V rounded to bf16 (nearest-even)."""
    X = bf16_to_f64(x)
    W = bf16_to_f64(w_qkv)
    T = X.shape[0]
    Y = X @ W.T                                   # [T][(Hq + 2 Hkv) D]
    q = np.zeros((T, Hq, D))
    cos = np.asarray(rope_cos, dtype=np.float64)
    sin = np.asarray(rope_sin, dtype=np.float64)
    kc = np.zeros((T, Hkv, D))
    vc = np.zeros((T, Hkv, D))
    for b in range(len(node_offsets) - 1):
        s0, s1 = int(node_offsets[b]), int(node_offsets[b + 1])
        P = int(prefix_len[b])
        par = np.asarray(parent[s0:s1])
        depth = np.zeros(s1 - s0, dtype=np.int64)
        for i in range(1, s1 - s0):
            depth[i] = depth[par[i]] + 1
        for i in range(s1 - s0):
            t = s0 + i
            pos = P + int(depth[i])
            for h in range(Hq):
                q[t, h] = rope_rotate(Y[t, h * D:(h + 1) * D], cos[pos], sin[pos])
            for g in range(Hkv):
                off = (Hq + g) * D
                kc[t, g] = rope_rotate(Y[t, off:off + D], cos[pos], sin[pos])
                off = (Hq + Hkv + g) * D
                vc[t, g] = Y[t, off:off + D]
            slot = P + i
            pg, ro = int(page_table[b, slot // page_size]), slot % page_size
            k_cache[pg, ro] = _f64_to_bf16_bits(kc[t])
            v_cache[pg, ro] = _f64_to_bf16_bits(vc[t])
    return q, kc, vc


def _f64_to_bf16_bits(a):
    """Round float64 values to nearest-even bf16 through fp32 (round to fp32
    first, then to bf16) -- only used to place oracle values in a bf16 cache."""
    f = np.asarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u >> 16) & 1) + 0x7FFF
    return ((u + r) >> 16).astype(np.uint16)
