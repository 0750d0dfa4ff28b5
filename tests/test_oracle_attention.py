"""Pins for the fp64 tree-attention oracle.

Definition followed (JetSpec README, "JetSpec / Overview"): one forward pass
under a tree-causal mask, i.e. node i attends to the prefix plus its own
root-to-i path exactly as causal attention over that sequence would.
"""
import math

import numpy as np
import pytest

import oracle
from helpers import (ancestor_matrix, bf16, dense_tree_attention, f64, logical_rows,
                     run_oracle_attention, small_case)
from tree_verification_jsv_b200 import synth


def test_matches_dense_masked_attention_on_random_trees():
    rng = np.random.default_rng(5)
    parents = [synth.tiny_tree(rng, 11, 4, 3), synth.tiny_tree(rng, 6, 3, 2), np.array([-1])]
    case = small_case(parents, [37, 0, 16], Hq=6, Hkv=2, D=16, seed=1)
    got = run_oracle_attention(case)
    ref = dense_tree_attention(case)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_chain_tree_equals_causal_attention():
    # a chain tree is ordinary decoding: node i sees slots 0..P+i
    N, P, D = 9, 21, 8
    case = small_case([np.arange(-1, N - 1)], [P], Hq=2, Hkv=1, D=D, seed=2)
    got = run_oracle_attention(case)
    K = logical_rows(case["k_cache"], case["page_table"], 0, P + N)[:, 0]
    V = logical_rows(case["v_cache"], case["page_table"], 0, P + N)[:, 0]
    L = P + N
    causal = np.tril(np.ones((L, L), dtype=bool))
    for h in range(2):
        Q = np.zeros((L, D))
        Q[P:] = f64(case["q"][:, h])
        S = case["scale"] * Q @ K.T
        S = np.where(causal, S, -np.inf)
        W = np.exp(S - S.max(axis=1, keepdims=True))
        W /= W.sum(axis=1, keepdims=True)
        O = W @ V
        assert np.max(np.abs(got[:, h] - O[P:])) < 1e-12


def test_single_node_no_prefix_returns_root_value_exactly():
    case = small_case([np.array([-1])], [0], Hq=2, Hkv=1, D=16, seed=3)
    got = run_oracle_attention(case)
    v = f64(case["v_cache"].reshape(-1, 1, 16)[int(case["page_table"][0, 0]) * 16])[0]
    for h in range(2):
        assert np.array_equal(got[0, h], v)


def test_identical_keys_give_mean_of_visible_values():
    parents = [np.array([-1, 0, 0, 1, 3, 2])]
    P = 19
    case = small_case(parents, [P], Hq=2, Hkv=1, D=16, seed=4)
    kc = case["k_cache"].copy()
    kc[:] = kc.reshape(-1, 16)[0]            # every cache row has the same key
    case["k_cache"] = kc
    got = run_oracle_attention(case)
    V = logical_rows(case["v_cache"], case["page_table"], 0, P + 6)[:, 0]
    A = ancestor_matrix(parents[0])
    for i in range(6):
        vis = list(range(P)) + [P + j for j in range(6) if A[i, j]]
        mean = V[vis].mean(axis=0)
        assert np.max(np.abs(got[i, 0] - mean)) < 1e-15
        assert np.max(np.abs(got[i, 1] - mean)) < 1e-15


def test_hand_worked_two_key_example():
    # tests/golden/attention_two_keys.txt: scores 0 and ln 3 give weights 1/4, 3/4
    spec = dict(l.split("=", 1) for l in open(
        __file__.replace("test_oracle_attention.py", "golden/attention_two_keys.txt"))
        .read().split("\n") if "=" in l and not l.startswith("#"))
    D = 2
    case = small_case([np.array([-1])], [1], Hq=1, Hkv=1, D=D, seed=0)
    kc = np.zeros_like(case["k_cache"])
    vc = np.zeros_like(case["v_cache"])
    pg = int(case["page_table"][0, 0])
    kc[pg, 0, 0] = bf16([0.0, 0.0])
    kc[pg, 1, 0] = bf16([1.0, 0.0])
    vc[pg, 0, 0] = bf16([float(x) for x in spec["v0"].split(",")])
    vc[pg, 1, 0] = bf16([float(x) for x in spec["v1"].split(",")])
    case.update(k_cache=kc, v_cache=vc, q=bf16(np.array([[[1.0, 0.0]]])),
                scale=float(np.float32(math.log(3.0))))
    got = run_oracle_attention(case)[0, 0]
    want = np.array([float(x) for x in spec["out"].split(",")])
    assert np.max(np.abs(got - want)) < 1e-7


def test_non_ancestor_kv_does_not_matter():
    parents = [np.array([-1, 0, 0, 1, 1, 2, 5])]
    P = 30
    case = small_case(parents, [P], Hq=4, Hkv=2, D=16, seed=6)
    base = run_oracle_attention(case)
    A = ancestor_matrix(parents[0])
    i = 3                                      # path 0-1-3; nodes 2,4,5,6 are not ancestors
    for j in [2, 4, 5, 6]:
        assert not A[i, j]
        kc, vc = case["k_cache"].copy(), case["v_cache"].copy()
        s = P + j
        pg, off = int(case["page_table"][0, s // 16]), s % 16
        kc[pg, off] ^= np.uint16(0x1234)
        vc[pg, off] ^= np.uint16(0x0F0F)
        got = run_oracle_attention(dict(case, k_cache=kc, v_cache=vc))
        assert np.array_equal(got[i], base[i])
        # ...but it does change the node that owns it
        assert not np.array_equal(got[j], base[j])


def test_relabelling_permutes_outputs():
    # same tree in two topological orders: outputs follow the relabelling
    par_a = np.array([-1, 0, 0, 1, 2, 2, 4])
    perm = np.array([0, 2, 1, 5, 4, 3, 6])      # new label of old node
    inv = np.argsort(perm)
    par_b = np.full(7, -1)
    for old in range(1, 7):
        par_b[perm[old]] = perm[par_a[old]]
    assert all(par_b[i] < i for i in range(1, 7))
    P = 17
    ca = small_case([par_a], [P], Hq=2, Hkv=1, D=16, seed=7, identity=True)
    cb = dict(ca)
    kc, vc, q = ca["k_cache"].copy(), ca["v_cache"].copy(), ca["q"].copy()
    flat_k, flat_v = kc.reshape(-1, 1, 16), vc.reshape(-1, 1, 16)
    src_k, src_v = ca["k_cache"].reshape(-1, 1, 16), ca["v_cache"].reshape(-1, 1, 16)
    for old in range(7):
        flat_k[P + perm[old]] = src_k[P + old]
        flat_v[P + perm[old]] = src_v[P + old]
        q[perm[old]] = ca["q"][old]
    cb.update(parent=par_b.astype(np.int32), k_cache=kc, v_cache=vc, q=q)
    oa, ob = run_oracle_attention(ca), run_oracle_attention(cb)
    for old in range(7):
        assert np.array_equal(oa[old], ob[perm[old]])
    assert inv is not None


def test_page_permutation_is_invisible():
    parents = [synth.tiny_tree(np.random.default_rng(8), 12, 5, 3)]
    a = small_case(parents, [53], Hq=2, Hkv=1, D=16, seed=9, identity=True)
    b = dict(a)
    rng = np.random.default_rng(10)
    perm = rng.permutation(a["num_pages"])
    kc = np.empty_like(a["k_cache"])
    vc = np.empty_like(a["v_cache"])
    kc[perm] = a["k_cache"]
    vc[perm] = a["v_cache"]
    table = a["page_table"].copy()
    m = table >= 0
    table[m] = perm[table[m]]
    b.update(k_cache=kc, v_cache=vc, page_table=table)
    assert np.array_equal(run_oracle_attention(a), run_oracle_attention(b))


def test_gqa_head_mapping():
    # query head h reads kv head h // G: zeroing kv head 1's values zeroes heads 2,3 only
    case = small_case([np.array([-1, 0, 1])], [20], Hq=4, Hkv=2, D=16, seed=11)
    vc = case["v_cache"].copy()
    vc[:, :, 1, :] = 0
    got = run_oracle_attention(dict(case, v_cache=vc))
    assert np.all(got[:, 2:] == 0)
    assert np.all(np.abs(got[:, :2]).sum(axis=-1) > 0)


def test_row_subset_matches_full():
    case = small_case([synth.tiny_tree(np.random.default_rng(12), 9, 4, 3)], [40], seed=12)
    full = run_oracle_attention(case)
    rows = np.array([[0, 0], [8, 3], [4, 1]])
    sub = run_oracle_attention(case, rows=rows)
    for r, (t, h) in enumerate(rows):
        assert np.array_equal(sub[r], full[t, h])


def test_malformed_tree_is_rejected():
    case = small_case([np.array([-1, 0, 1])], [4], Hq=2, Hkv=1, D=16, seed=13)
    case["parent"] = np.array([-1, 2, 1], dtype=np.int32)   # cycle 1 <-> 2
    with pytest.raises(ValueError):
        run_oracle_attention(case)
