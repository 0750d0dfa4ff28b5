"""Seeded synthetic inputs for the one-forward tree verification step.

This module holds random draws and the recipe for the *shape* of the inputs
only: tree shapes, paging, bf16 value draws and the per-node token-planting
coin flips.  It contains none of the verification arithmetic (no attention,
no logits, no argmax, no walk, no copy).  Where a token must equal the
target's argmax of its parent, the argmax is an *input* to ``plant_tokens``;
the caller obtains it elsewhere.

Workload shapes stand in for the pages' Qwen3-8B and Qwen3-30B-A3B targets
at tree budgets of 64-512 nodes (JetSpec README, "Inference engine" and
"Evaluation" sections: ``tree_depth``, ``tree_width``, ``budget``).  The pages
measure on math/code/chat datasets; synthetic draws stand in for them.

Every array is drawn from numpy PCG64 streams keyed by (seed, stream id,
extra keys).  Large arrays are drawn in fixed blocks of ``_BLOCK`` elements,
each block with its own key, so the bytes do not depend on how many threads
draw them.  Floating values are drawn in fp32, scaled, and rounded to
nearest-even bf16; bf16 tensors are carried as ``uint16`` bit patterns.
"""
from __future__ import annotations

import heapq
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

PAGE_SIZE = 16
_BLOCK = 1 << 22

_STREAM = {
    "shape": 1, "tree": 2, "q": 3, "k": 4, "v": 5, "hidden": 6, "w": 7,
    "tok_flag": 8, "tok_uniform": 9, "pages": 10, "prefix": 11,
    "hidden_redraw": 12, "match_p": 13,
}


def _rng(seed: int, name: str, *extra: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), _STREAM[name], *[int(e) for e in extra]])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to nearest-even bf16, returned as uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, name: str, n: int, scale: float, *extra: int) -> np.ndarray:
    """``n`` draws of N(0,1)*scale rounded to bf16 bits, block-keyed."""
    out = np.empty(n, dtype=np.uint16)
    nblk = (n + _BLOCK - 1) // _BLOCK
    s = np.float32(scale)

    def one(bi: int) -> None:
        lo = bi * _BLOCK
        hi = min(n, lo + _BLOCK)
        x = _rng(seed, name, *extra, bi).standard_normal(hi - lo, dtype=np.float32)
        x *= s
        out[lo:hi] = f32_to_bf16_bits(x)

    if nblk <= 1:
        for bi in range(nblk):
            one(bi)
    else:
        with ThreadPoolExecutor(min(nblk, os.cpu_count() or 1)) as ex:
            list(ex.map(one, range(nblk)))
    return out


# --------------------------------------------------------------------------
# Tree shapes
# --------------------------------------------------------------------------

def tiny_tree(rng: np.random.Generator, n: int, max_depth: int, max_children: int) -> np.ndarray:
    """Random topological tree: node i>0 picks a uniform parent among earlier
    nodes of depth < max_depth with fewer than max_children children."""
    parent = np.full(n, -1, dtype=np.int32)
    depth = np.zeros(n, dtype=np.int32)
    nchild = np.zeros(n, dtype=np.int32)
    for i in range(1, n):
        cand = [j for j in range(i) if depth[j] < max_depth and nchild[j] < max_children]
        p = cand[int(rng.integers(len(cand)))]
        parent[i] = p
        depth[i] = depth[p] + 1
        nchild[p] += 1
    return parent


def budget_tree(rng: np.random.Generator, budget: int, max_depth: int, topk: int) -> np.ndarray:
    """Budgeted draft tree in BFS order.

    Shape recipe (a reading of the pages' ``accum_logp`` default: a
    breadth-first tree kept by cumulative log-probability under depth, width
    and budget): every node below ``max_depth`` offers ``topk`` ranked
    children whose edge log-scores are the logs of ``topk`` normalised
    uniforms sorted in descending order.  The rank-0 chain down to
    ``max_depth`` is always kept so the stated depth is realised; the rest of
    the budget is filled best-first by cumulative score.  Cumulative scores
    only fall along a path, so the kept set is ancestor-closed.  Nodes are
    then relabelled breadth-first (children in rank order).
    """
    par: list[int] = [-1]
    dep: list[int] = [0]
    rank: list[int] = [0]
    score: list[float] = [0.0]
    edge: list[np.ndarray] = []

    def edges_for(node: int) -> None:
        u = rng.random(topk) + 1e-12
        p = np.sort(u / u.sum())[::-1]
        edge.append(np.log(p))

    taken: set[tuple[int, int]] = set()
    heap: list[tuple[float, int, int, int]] = []
    counter = 0

    def add(parent: int, r: int) -> int:
        nonlocal counter
        node = len(par)
        par.append(parent)
        dep.append(dep[parent] + 1)
        rank.append(r)
        score.append(score[parent] + float(edge[parent][r]))
        taken.add((parent, r))
        edges_for(node)
        return node

    edges_for(0)
    cur = 0
    while dep[cur] < max_depth and len(par) < budget:
        cur = add(cur, 0)
    for node in range(len(par)):
        if dep[node] < max_depth:
            for r in range(topk):
                if (node, r) not in taken:
                    heapq.heappush(heap, (-(score[node] + float(edge[node][r])), counter, node, r))
                    counter += 1
    while len(par) < budget and heap:
        _, _, p, r = heapq.heappop(heap)
        node = add(p, r)
        if dep[node] < max_depth:
            for rr in range(topk):
                heapq.heappush(heap, (-(score[node] + float(edge[node][rr])), counter, node, rr))
                counter += 1

    n = len(par)
    children: list[list[int]] = [[] for _ in range(n)]
    for i in range(1, n):
        children[par[i]].append(i)
    order = [0]
    head = 0
    while head < len(order):
        x = order[head]
        head += 1
        order.extend(sorted(children[x], key=lambda c: rank[c]))
    new_of = np.empty(n, dtype=np.int64)
    new_of[np.asarray(order)] = np.arange(n)
    parent = np.full(n, -1, dtype=np.int32)
    for old in range(1, n):
        parent[new_of[old]] = new_of[par[old]]
    return parent


def depths(parent: np.ndarray) -> np.ndarray:
    d = np.zeros(len(parent), dtype=np.int32)
    for i in range(1, len(parent)):
        d[i] = d[parent[i]] + 1
    return d


# --------------------------------------------------------------------------
# Configurations
# --------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    D: int
    d: int
    V: int
    prefix_len: np.ndarray          # int32 [B]
    node_offsets: np.ndarray        # int32 [B+1]
    parent: np.ndarray              # int32 [T], request-local indices
    match_p: np.ndarray             # float64 [B]
    page_table: np.ndarray          # int32 [B, max_pages_per_req], -1 = unmapped
    num_pages: int
    q: np.ndarray = field(repr=False, default=None)        # uint16 [T, Hq, D]
    k_cache: np.ndarray = field(repr=False, default=None)  # uint16 [num_pages, 16, Hkv, D]
    v_cache: np.ndarray = field(repr=False, default=None)
    hidden: np.ndarray = field(repr=False, default=None)   # uint16 [T, d]
    w: np.ndarray = field(repr=False, default=None)        # uint16 [V, d]
    tok_flag: np.ndarray = field(repr=False, default=None)     # bool [T]
    tok_uniform: np.ndarray = field(repr=False, default=None)  # int32 [T]
    redraws: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.node_offsets[-1])

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(D), as the fp32 value both sides use."""
        return float(np.float32(1.0 / math.sqrt(self.D)))

    @property
    def max_nodes(self) -> int:
        return int(np.max(np.diff(self.node_offsets)))

    @property
    def max_prefix(self) -> int:
        return int(np.max(self.prefix_len))

    @property
    def max_pages_per_req(self) -> int:
        return int(self.page_table.shape[1])

    def request_nodes(self, b: int) -> slice:
        return slice(int(self.node_offsets[b]), int(self.node_offsets[b + 1]))


# name -> (B, Hq, Hkv, D, d, V)
SHAPES = {
    "tiny": (1, 2, 1, 64, 256, 1024),
    "8b_64": (1, 32, 8, 128, 4096, 151936),
    "8b_256": (1, 32, 8, 128, 4096, 151936),
    "ragged16": (16, 32, 8, 128, 4096, 151936),
    "30b_512x4": (4, 32, 4, 128, 2048, 151936),
}
CONFIG_INDEX = {"tiny": 0, "8b_64": 1, "8b_256": 2, "ragged16": 3, "30b_512x4": 4}


def default_seed(name: str) -> int:
    return 1000 + CONFIG_INDEX[name]


def _trees_and_prefix(name: str, seed: int):
    sh = _rng(seed, "shape")
    if name == "tiny":
        return [tiny_tree(_rng(seed, "tree", 0), 16, 5, 3)], [128], [0.7]
    if name == "8b_64":
        return [budget_tree(_rng(seed, "tree", 0), 64, 8, 4)], [2048], [0.7]
    if name == "8b_256":
        return [budget_tree(_rng(seed, "tree", 0), 256, 16, 8)], [16384], [0.8]
    if name == "30b_512x4":
        return ([budget_tree(_rng(seed, "tree", b), 512, 16, 8) for b in range(4)],
                [32768] * 4, [0.8] * 4)
    if name == "ragged16":
        trees, pre, ps = [], [], []
        for b in range(16):
            n = int(sh.integers(32, 129))
            dep = int(sh.integers(4, 13))
            trees.append(budget_tree(_rng(seed, "tree", b), n, dep, 4))
            pre.append(int(sh.integers(512, 8193)))
            ps.append(float(sh.uniform(0.4, 0.9)))
        return trees, pre, ps
    raise KeyError(name)


def make_paging(seed: int, prefix_len, nodes, spare_pages: int = 2, identity: bool = False):
    """Page table covering slots [0, P_b + N_b) of every request, with the
    physical pages in a seeded random permutation (non-contiguous)."""
    need = [(p + n + PAGE_SIZE - 1) // PAGE_SIZE for p, n in zip(prefix_len, nodes)]
    num_pages = int(sum(need)) + spare_pages
    perm = np.arange(num_pages) if identity else _rng(seed, "pages").permutation(num_pages)
    maxp = max(need)
    table = np.full((len(need), maxp), -1, dtype=np.int32)
    at = 0
    for b, k in enumerate(need):
        table[b, :k] = perm[at:at + k]
        at += k
    return table, num_pages


def make_workload(name: str, seed: int | None = None, *, identity_pages: bool = False,
                  q_scale: float = 1.0, values: bool = True, lmhead: bool = True,
                  redraws: dict | None = None) -> Workload:
    """Build one named workload.  ``q_scale`` multiplies Q before rounding
    (a "sharp attention" variant); ``redraws`` maps global node index -> the
    number of times its hidden row was redrawn by margin certification."""
    if seed is None:
        seed = default_seed(name)
    B, Hq, Hkv, D, d, V = SHAPES[name]
    trees, prefix, ps = _trees_and_prefix(name, seed)
    nodes = [len(t) for t in trees]
    offs = np.zeros(B + 1, dtype=np.int32)
    offs[1:] = np.cumsum(nodes)
    table, num_pages = make_paging(seed, prefix, nodes, identity=identity_pages)
    wl = Workload(name=name, seed=seed, B=B, Hq=Hq, Hkv=Hkv, D=D, d=d, V=V,
                  prefix_len=np.asarray(prefix, dtype=np.int32), node_offsets=offs,
                  parent=np.concatenate(trees).astype(np.int32),
                  match_p=np.asarray(ps, dtype=np.float64),
                  page_table=table, num_pages=num_pages, redraws=dict(redraws or {}))
    T = wl.T
    fl = _rng(seed, "tok_flag").random(T)
    wl.tok_flag = np.zeros(T, dtype=bool)
    for b in range(B):
        sl = wl.request_nodes(b)
        wl.tok_flag[sl] = fl[sl] < ps[b]
        wl.tok_flag[sl.start] = False          # root token is never planted
    wl.tok_uniform = _rng(seed, "tok_uniform").integers(0, V, T).astype(np.int32)
    if values:
        wl.q = normal_bf16(seed, "q", T * Hq * D, q_scale / math.sqrt(D)).reshape(T, Hq, D)
        kv = num_pages * PAGE_SIZE * Hkv * D
        wl.k_cache = normal_bf16(seed, "k", kv, 1.0 / math.sqrt(D)).reshape(num_pages, PAGE_SIZE, Hkv, D)
        wl.v_cache = normal_bf16(seed, "v", kv, 1.0 / math.sqrt(D)).reshape(num_pages, PAGE_SIZE, Hkv, D)
    if lmhead:
        wl.w = normal_bf16(seed, "w", V * d, 1.0 / math.sqrt(d)).reshape(V, d)
        wl.hidden = hidden_rows(seed, T, d, wl.redraws)
    return wl


def hidden_rows(seed: int, T: int, d: int, redraws: dict | None = None) -> np.ndarray:
    """Hidden states [T, d]; a node listed in ``redraws`` with count r takes
    its row from sub-stream (node, r) instead of the base draw."""
    h = normal_bf16(seed, "hidden", T * d, 1.0 / math.sqrt(d)).reshape(T, d)
    for t, r in (redraws or {}).items():
        t, r = int(t), int(r)
        if r > 0:
            h[t] = normal_bf16(seed, "hidden_redraw", d, 1.0 / math.sqrt(d), t, r)
    return h


def plant_tokens(wl: Workload, argmax: np.ndarray) -> np.ndarray:
    """Tree tokens: a non-root node whose coin came up carries its parent's
    argmax token (given), every other node a uniform token in [0, V)."""
    argmax = np.asarray(argmax, dtype=np.int64)
    tok = wl.tok_uniform.astype(np.int32).copy()
    for b in range(wl.B):
        sl = wl.request_nodes(b)
        base = sl.start
        for i in range(1, sl.stop - sl.start):
            t = base + i
            if wl.tok_flag[t]:
                tok[t] = argmax[base + int(wl.parent[t])]
    return tok


# --------------------------------------------------------------------------
# Draft-head top-k per depth (input of the budgeted tree construction)
# --------------------------------------------------------------------------

def draft_topk(seed: int, B: int, D: int, k: int, V: int):
    """Synthetic draft-head output for ``B`` requests: for each depth 1..D,
    ``k`` candidate tokens with log-probabilities sorted in descending order
    (logs of ``k`` normalised uniforms), plus a root token per request.
    Returns (logp float32 [B][D][k], tokens int32 [B][D][k], root int32 [B])."""
    g = _rng(seed, "tree", 10_000)
    u = g.random((B, D, k)) + 1e-6
    p = np.sort(u / u.sum(axis=2, keepdims=True), axis=2)[:, :, ::-1]
    logp = np.log(p).astype(np.float32)
    tok = g.integers(0, V, (B, D, k)).astype(np.int32)
    root = g.integers(0, V, B).astype(np.int32)
    return np.ascontiguousarray(logp), tok, root
