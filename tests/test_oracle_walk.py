"""Pins for the greedy accept walk (JetSpec README, "JetSpec / Overview": the
accepted path follows the target's own logits, so decoding is lossless;
"tokens per forward" in its engine example counts accepted tokens + 1)."""
import numpy as np

import oracle
from tree_verification_jsv_b200 import synth


def _greedy_decode(parent, tokens, argmax, limit=10_000):
    """Independent simulator: run the target token by token.  The context
    after emitting y_1..y_k is a tree node when the draft covers it; the target
    then emits argmax at that node.  Recursion over an explicit child map."""
    kids = {}
    for c in range(1, len(parent)):
        kids.setdefault(int(parent[c]), []).append(c)

    def step(node, emitted):
        y = int(argmax[node])
        emitted.append(y)
        if len(emitted) > limit:
            return emitted
        covering = [c for c in sorted(kids.get(node, [])) if int(tokens[c]) == y]
        return step(covering[0], emitted) if covering else emitted
    return step(0, [])


def _brute_longest(parent, tokens, argmax):
    """Longest root-started path whose every edge token equals the target's
    choice at the edge's parent (all paths enumerated)."""
    n = len(parent)
    best = [0]
    for leaf in range(n):
        path = []
        j = leaf
        while j != -1:
            path.append(j)
            j = int(parent[j])
        path = path[::-1]
        k = 1
        while k < len(path) and int(tokens[path[k]]) == int(argmax[path[k - 1]]):
            k += 1
        if k > len(best):
            best = path[:k]
    return best


def test_chain_all_match():
    n = 9
    parent = np.arange(-1, n - 1)
    argmax = np.arange(100, 100 + n)
    tokens = np.concatenate([[7], argmax[:-1]])
    path, a, bonus = oracle.accept_path(parent, tokens, argmax)
    assert path == list(range(n)) and a == n - 1 and bonus == argmax[-1]


def test_root_without_matching_child():
    parent = np.array([-1, 0, 0, 1])
    tokens = np.array([5, 1, 2, 3])
    argmax = np.array([9, 9, 9, 9])
    assert oracle.accept_path(parent, tokens, argmax) == ([0], 0, 9)


def test_second_sibling_branch_is_taken():
    parent = np.array([-1, 0, 0, 2, 1])
    tokens = np.array([0, 11, 12, 13, 14])
    argmax = np.array([12, 0, 13, 40, 0])
    assert oracle.accept_path(parent, tokens, argmax) == ([0, 2, 3], 2, 40)


def test_duplicate_siblings_take_smaller_index():
    parent = np.array([-1, 0, 0, 1, 2])
    tokens = np.array([0, 8, 8, 3, 3])
    argmax = np.array([8, 3, 3, 1, 2])
    assert oracle.accept_path(parent, tokens, argmax) == ([0, 1, 3], 2, 1)
    # the larger duplicate is used only if the smaller one is absent
    tokens2 = np.array([0, 9, 8, 3, 3])
    assert oracle.accept_path(parent, tokens2, argmax) == ([0, 2, 4], 2, 2)


def test_deep_branch_beside_shallow_full_match():
    # root -> 1 (matches, leaf) and root -> 2 -> 3 -> 4 (does not match at 2)
    parent = np.array([-1, 0, 0, 2, 3])
    tokens = np.array([0, 5, 6, 7, 8])
    argmax = np.array([5, 77, 7, 8, 9])
    assert oracle.accept_path(parent, tokens, argmax) == ([0, 1], 1, 77)


def test_matches_brute_force_and_greedy_decoding_on_random_trees():
    rng = np.random.default_rng(3)
    for trial in range(300):
        depth, width = int(rng.integers(1, 10)), int(rng.integers(1, 5))
        cap = sum(width ** k for k in range(depth + 1))
        n = min(int(rng.integers(1, 40)), cap)
        parent = synth.tiny_tree(rng, n, depth, width)
        V = 1000
        argmax = rng.integers(0, V, n)
        tokens = rng.integers(0, V, n)
        for c in range(1, n):
            if rng.random() < 0.7:
                tokens[c] = argmax[parent[c]]
        # distinct tokens among siblings makes the longest path unique
        seen = {}
        for c in range(1, n):
            key = (int(parent[c]), int(tokens[c]))
            if key in seen:
                tokens[c] = V + c
            seen[key] = c
        path, a, bonus = oracle.accept_path(parent, tokens, argmax)
        assert path == _brute_longest(parent, tokens, argmax)
        emitted = [int(tokens[j]) for j in path[1:]] + [bonus]
        assert emitted == _greedy_decode(parent, tokens, argmax)[:a + 1]
        assert len(_greedy_decode(parent, tokens, argmax)) == a + 1


def test_greedy_decoding_with_duplicates():
    rng = np.random.default_rng(4)
    for trial in range(200):
        n = int(rng.integers(2, 30))
        parent = synth.tiny_tree(rng, n, 6, 4)
        argmax = rng.integers(0, 4, n)            # tiny vocab: many duplicates
        tokens = rng.integers(0, 4, n)
        path, a, bonus = oracle.accept_path(parent, tokens, argmax)
        emitted = [int(tokens[j]) for j in path[1:]] + [bonus]
        assert emitted == _greedy_decode(parent, tokens, argmax)
        # every step took the smallest matching child
        for k in range(1, len(path)):
            m = [c for c in range(n) if parent[c] == path[k - 1] and tokens[c] == argmax[path[k - 1]]]
            assert path[k] == min(m)
