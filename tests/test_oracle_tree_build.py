"""Pins for the accum_logp tree-construction oracle (JetSpec README,
"Evaluation": the default tree keeps the best nodes by cumulative
log-probability under depth, width and budget, breadth-first)."""
import itertools

import numpy as np
import pytest

import oracle


def _draft(rng, D, k, V=1000, ties=False):
    u = rng.random((D, k)) + 1e-3
    if ties:
        u = np.round(u * 4) + 1                  # few distinct values: many exact ties
    p = np.sort(u / u.sum(axis=1, keepdims=True), axis=1)[:, ::-1]
    return np.log(p).astype(np.float32), rng.integers(0, V, (D, k))


def _brute(logp, toks, root, budget):
    """Every rank path up to depth D, scored by fp32 running sums, sorted by
    the total order, best `budget` kept (the definition, by enumeration)."""
    D, k = logp.shape
    nodes = [((), np.float32(0.0))]
    for m in range(1, D + 1):
        for path in itertools.product(range(k), repeat=m):
            s = np.float32(0.0)
            for i, r in enumerate(path):
                s = np.float32(s + logp[i][r])
            nodes.append((path, s))
    def code(path):
        c = 0
        for r in path:
            c = c * k + r
        return c
    nodes.sort(key=lambda x: (-float(x[1]), len(x[0]), code(x[0])))
    return {p: s for p, s in nodes[:budget]}


def _paths(tree):
    """Rank-free view: map each node to its token path from the root."""
    out = []
    for i in range(len(tree["parent"])):
        path, j = [], i
        while j != -1:
            path.append(j)
            j = tree["parent"][j]
        out.append(tuple(path[::-1]))
    return out


@pytest.mark.parametrize("D,k,budget,ties", [(3, 3, 10, False), (4, 2, 12, False), (3, 4, 30, False),
                                             (5, 3, 50, False), (3, 3, 14, True), (4, 3, 40, True),
                                             (2, 2, 100, False)])
def test_matches_exhaustive_enumeration(D, k, budget, ties):
    rng = np.random.default_rng(D * 100 + k * 10 + budget)
    logp, toks = _draft(rng, D, k, ties=ties)
    tree = oracle.accum_logp_tree(logp, toks, 7, budget)
    want = _brute(logp, toks, 7, budget)
    n = len(tree["parent"])
    assert n == min(budget, sum(k ** m for m in range(D + 1)))
    # rebuild every node's rank path from codes and depths and compare sets
    got = {}
    for i in range(n):
        c, d = int(tree["code"][i]), int(tree["depth"][i])
        path = []
        for _ in range(d):
            path.append(c % k)
            c //= k
        got[tuple(path[::-1])] = tree["score"][i]
    assert set(got) == set(want)
    for pth, s in got.items():
        assert s == want[pth]


def test_structure_bfs_closure_tokens_scores():
    rng = np.random.default_rng(1)
    D, k, budget = 16, 8, 256
    logp, toks = _draft(rng, D, k, V=151936)
    t = oracle.accum_logp_tree(logp, toks, 42, budget)
    par, dep, sc, tok = t["parent"], t["depth"], t["score"], t["tokens"]
    assert len(par) == budget and par[0] == -1 and tok[0] == 42
    assert np.all(par[1:] < np.arange(1, budget))            # topological
    assert np.all(np.diff(dep) >= 0)                         # breadth-first levels
    assert np.all(dep[1:] == dep[par[1:]] + 1)
    codes = t["code"].astype(object)
    for i in range(1, budget):
        r = int(codes[i]) % k
        assert codes[i] == codes[par[i]] * k + r
        assert sc[i] == np.float32(sc[par[i]] + logp[dep[i] - 1][r])   # running fp32 sum
        assert tok[i] == toks[dep[i] - 1][r]
        assert sc[i] <= sc[par[i]]
        if r > 0:                                            # sibling-closed
            sib = [j for j in range(1, budget) if par[j] == par[i] and int(codes[j]) % k == r - 1]
            assert len(sib) == 1
    # children of one parent appear in rank order, parents in BFS order
    for d in range(1, dep.max() + 1):
        lvl = np.where(dep == d)[0]
        keys = [(par[i], int(codes[i]) % k) for i in lvl]
        assert keys == sorted(keys)


def test_budget_larger_than_tree_and_degenerate_sizes():
    logp = np.log(np.array([[0.6, 0.4], [0.7, 0.3]], dtype=np.float32))
    toks = np.array([[1, 2], [3, 4]])
    t = oracle.accum_logp_tree(logp, toks, 0, 1000)
    assert len(t["parent"]) == 1 + 2 + 4
    t1 = oracle.accum_logp_tree(logp, toks, 5, 1)
    assert list(t1["parent"]) == [-1] and list(t1["tokens"]) == [5]
    # a hand-worked case: scores log .6=-.51, log .4=-.92, .6*.7, .6*.3, .4*.7 ...
    t3 = oracle.accum_logp_tree(logp, toks, 0, 4)
    # best three non-root: (0) .6, (0,0) .42, (1) .4
    assert list(t3["depth"]) == [0, 1, 1, 2]
    assert list(t3["tokens"]) == [0, 1, 2, 3]
    assert list(t3["parent"]) == [-1, 0, 0, 1]
