"""Pins for the accepted-path KV compaction (paged KV in the JetSpec engine,
README "JetSpec / Quick Start"): after the step, the accepted path's K/V rows
must sit in contiguous slots P..P+a so the next step sees an ordinary prefix."""
import numpy as np

import oracle
from helpers import small_case
from tree_verification_jsv_b200 import synth


def _closed_form_check(before, after, table, P, path, n_slots_total):
    """cache'[P+k] = cache[P+path[k]] for k <= a; every other byte unchanged."""
    flat_b = before.reshape(-1, before.shape[2], before.shape[3])
    flat_a = after.reshape(-1, after.shape[2], after.shape[3])
    touched = set()
    for k, j in enumerate(path):
        dst = P + k
        src = P + j
        d = table[dst // 16] * 16 + dst % 16
        s = table[src // 16] * 16 + src % 16
        assert np.array_equal(flat_a[d], flat_b[s])
        touched.add(int(d))
    rest = np.array([r for r in range(flat_b.shape[0]) if r not in touched])
    assert np.array_equal(flat_a[rest], flat_b[rest])


def test_closed_form_on_random_paths():
    rng = np.random.default_rng(0)
    for trial in range(30):
        n = int(rng.integers(1, 60))
        P = int(rng.integers(0, 70))
        parent = synth.tiny_tree(rng, n, 20, 3)
        case = small_case([parent], [P], Hq=2, Hkv=2, D=8, seed=trial)
        # a random root-to-node path
        leaf = int(rng.integers(0, n))
        path = []
        j = leaf
        while j != -1:
            path.append(j)
            j = int(parent[j])
        path = path[::-1]
        kb, vb = case["k_cache"].copy(), case["v_cache"].copy()
        k, v = case["k_cache"].copy(), case["v_cache"].copy()
        new_len = oracle.kv_compact(k, v, case["page_table"], case["prefix_len"], [path])
        assert list(new_len) == [P + len(path)]
        _closed_form_check(kb, k, case["page_table"][0], P, path, None)
        _closed_form_check(vb, v, case["page_table"][0], P, path, None)


def test_zero_accepted_is_identity():
    case = small_case([np.array([-1, 0, 0])], [5], Hq=2, Hkv=1, D=8, seed=1)
    k, v = case["k_cache"].copy(), case["v_cache"].copy()
    nl = oracle.kv_compact(k, v, case["page_table"], case["prefix_len"], [[0]])
    assert list(nl) == [6]
    assert np.array_equal(k, case["k_cache"]) and np.array_equal(v, case["v_cache"])


def test_overlapping_moves_read_before_overwrite():
    # chain whose accepted path skips every other node: path[k] = 2k moves rows
    # onto slots that later steps would read if done in the wrong order
    n = 21
    parent = np.array([-1] + [max(0, i - 2) if i % 2 == 0 else i - 1 for i in range(1, n)])
    path = list(range(0, n, 2))
    assert all(parent[path[k]] == path[k - 1] for k in range(1, len(path)))
    case = small_case([parent], [13], Hq=2, Hkv=1, D=8, seed=2)
    k, v = case["k_cache"].copy(), case["v_cache"].copy()
    oracle.kv_compact(k, v, case["page_table"], case["prefix_len"], [path])
    _closed_form_check(case["k_cache"], k, case["page_table"][0], 13, path, None)


def test_ragged_batch_requests_are_independent():
    rng = np.random.default_rng(3)
    parents = [synth.tiny_tree(rng, n, 8, 3) for n in (5, 17, 1, 9)]
    case = small_case(parents, [3, 40, 0, 16], Hq=2, Hkv=2, D=8, seed=3)
    paths = []
    for p in parents:
        leaf = len(p) - 1
        path = []
        while leaf != -1:
            path.append(leaf)
            leaf = int(p[leaf])
        paths.append(path[::-1])
    k, v = case["k_cache"].copy(), case["v_cache"].copy()
    nl = oracle.kv_compact(k, v, case["page_table"], case["prefix_len"], paths)
    assert list(nl) == [P + len(pa) for P, pa in zip([3, 40, 0, 16], paths)]
    # request by request, on a fresh copy, gives the same bytes
    k2, v2 = case["k_cache"].copy(), case["v_cache"].copy()
    for b in range(4):
        oracle.kv_compact(k2, v2, case["page_table"][b:b + 1], case["prefix_len"][b:b + 1], [paths[b]])
    assert np.array_equal(k, k2) and np.array_equal(v, v2)
