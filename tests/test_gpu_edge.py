"""GPU edge cases through the C ABI: tiny and degenerate trees, ragged
prefixes that are not multiples of the page size, trees crossing page
boundaries, sharp attention, head-dim 64, G = 1 and G that does not divide a
row group, vocabulary and node counts
that are not tile multiples, and device-side error reporting."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import attention_close, bf16, dense_tree_attention, small_case
from tree_verification_jsv_b200 import jsv, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_jsv_b200 import build
    build.build()
    jsv.load()


def _dev_i32(x):
    return torch.as_tensor(np.ascontiguousarray(x, dtype=np.int32)).cuda()


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _batch(case, status, **over):
    offs = case["node_offsets"]
    n = np.diff(offs)
    dev = dict(page_table=_dev_i32(case["page_table"]), prefix_len=_dev_i32(case["prefix_len"]),
               node_offsets=_dev_i32(offs), parent=_dev_i32(case["parent"]))
    kw = dict(B=len(n), Hq=case["Hq"], Hkv=case["Hkv"], D=case["D"],
              max_pages_per_req=case["page_table"].shape[1], num_pages=case["num_pages"],
              total_nodes=int(offs[-1]), max_nodes=int(n.max()),
              max_prefix=int(max(case["prefix_len"])), dev_status=status, **dev)
    kw.update(over)
    return jsv.make_batch(**kw), dev


def run_attention(case, **over):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    batch, keep = _batch(case, status, **over)
    q = _dev_bf16(case["q"])
    k = _dev_bf16(case["k_cache"])
    v = _dev_bf16(case["v_cache"])
    T = int(case["node_offsets"][-1])
    out = torch.zeros((T, case["Hq"], case["D"]), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(256, jsv.jsv_tree_attention_workspace_size(batch)), dtype=torch.uint8, device="cuda")
    jsv.jsv_tree_attention(batch, q, k, v, case["scale"], out, ws)
    torch.cuda.synchronize()
    return synth.bf16_bits_to_f32(_bits(out)).astype(np.float64), int(status.item())


ATTN_CASES = {
    "single_node_no_prefix": ([np.array([-1])], [0], 4, 2, 128),
    "root_only_prefix_17": ([np.array([-1])], [17], 4, 2, 128),
    "chain_cross_pages": ([np.arange(-1, 40)], [29], 8, 2, 128),
    "ragged_three": ([synth.tiny_tree(np.random.default_rng(1), 23, 6, 3),
                      np.array([-1, 0]), synth.tiny_tree(np.random.default_rng(2), 70, 9, 4)],
                     [1, 0, 300], 8, 2, 128),
    "head_dim_64_g1": ([synth.tiny_tree(np.random.default_rng(3), 31, 5, 3)], [45], 4, 4, 64),
    "g8_long": ([synth.budget_tree(np.random.default_rng(4), 100, 10, 4)], [1500], 16, 2, 128),
    "max_nodes_512": ([synth.budget_tree(np.random.default_rng(5), 512, 16, 8)], [64], 2, 1, 64),
    # G that does not divide a 128-row group (Q staged by plain loads, rows
    # of one node split across CTA tiles)
    "g5_two_row_tiles": ([synth.budget_tree(np.random.default_rng(6), 60, 8, 4)], [700], 10, 2, 128),
    "g3_head_dim_64": ([synth.tiny_tree(np.random.default_rng(7), 50, 6, 3),
                        synth.tiny_tree(np.random.default_rng(8), 9, 3, 2)], [130, 33], 6, 2, 64),
    # a ragged batch: the two long requests take several KV splits (merged by
    # the combine kernel) while the short ones take one split each and are
    # written straight from the attention kernel
    "short_and_long_mix": ([np.arange(-1, 30)] + [synth.tiny_tree(np.random.default_rng(20 + i), 5 + i, 4, 3)
                                                  for i in range(18)] + [np.arange(-1, 9)],
                           [8000] + [50 + 7 * i for i in range(18)] + [5003], 8, 2, 128),
    # G = 16 (Q by TMA, 8 nodes per 128-row group), a prefix ending inside a
    # page and a 256-node tree whose tiles fall into more than one split
    "g16_tree_cut": ([synth.budget_tree(np.random.default_rng(9), 256, 16, 8)], [2077], 16, 1, 128),
    # 48 requests with prefixes from 16 to 1500 tokens and trees of 1 to 20
    # nodes: 384 (request, KV head) units, so the launch takes one split per
    # request and orders the units longest first
    # no GQA packing at head dimension 128 (G = 1: 128 nodes per row group)
    "g1_head_dim_128": ([synth.tiny_tree(np.random.default_rng(40), 150, 9, 3)], [300], 4, 4, 128),
    # more requests than the longest-first order takes (70 > 64): block-index
    # units, most of them single-tile requests, a few prefixes of zero
    "b70_block_order": ([synth.tiny_tree(np.random.default_rng(500 + i), 1 + i % 5, 3, 2) for i in range(70)],
                        [(37 * i) % 211 if i % 9 else 0 for i in range(70)], 4, 2, 64),
    "lpt_48_ragged": ([synth.tiny_tree(np.random.default_rng(300 + i), 1 + (7 * i) % 20, 4, 3) for i in range(48)],
                      [16 + (353 * i) % 1485 for i in range(48)], 16, 8, 64),
}


@pytest.mark.parametrize("name", list(ATTN_CASES))
@pytest.mark.parametrize("sharp", [False, True])
def test_attention_edge_cases(name, sharp):
    parents, pre, Hq, Hkv, D = ATTN_CASES[name]
    case = small_case(parents, pre, Hq=Hq, Hkv=Hkv, D=D, seed=11,
                      q_scale=4.0 * math.sqrt(D) if sharp else 1.0)
    got, st = run_attention(case)
    assert st == 0
    from helpers import run_oracle_attention
    attention_close(got, run_oracle_attention(case), name)


@pytest.mark.parametrize("seed", range(8))
def test_attention_random_geometry(seed):
    """Seeded random batches against the oracle: 1 to 70 requests (both unit
    orders and both one and several splits), G in {1, 2, 3, 4, 8, 16}, D in
    {64, 128}, prefixes from 0 to 2500 (page-aligned or not), trees of 1 to
    180 nodes of random shape, and sharp queries in half of them."""
    rng = np.random.default_rng(1000 + seed)
    G = (1, 2, 3, 4, 8, 16, 4, 8)[seed]
    B = (1, 2, 5, 17, 70, 3, 64, 1)[seed]
    D = (64, 128)[(seed + seed // 4) % 2]
    Hkv = int(rng.choice([1, 2])) if G >= 8 else int(rng.choice([1, 2, 4]))
    cap = 180 if B <= 5 else 24
    parents = []
    for _ in range(B):
        n = int(rng.integers(1, cap + 1))
        depth = int(rng.integers(max(1, math.ceil(math.log2(n + 1))), 13))   # room for n nodes at 2+ children
        parents.append(synth.tiny_tree(rng, n, depth, int(rng.integers(2, 5))))
    pre = [int(rng.choice([0, 16, 17, 255, 1024, int(rng.integers(0, 2500))])) for _ in range(B)]
    case = small_case(parents, pre, Hq=G * Hkv, Hkv=Hkv, D=D, seed=2000 + seed, q_scale=4.0 if seed % 2 else 1.0)
    got, st = run_attention(case)
    assert st == 0
    from helpers import run_oracle_attention
    attention_close(got, run_oracle_attention(case), f"random geometry {seed}")


def test_attention_workspace_reused_without_clearing():
    """One attention workspace, filled with garbage once, serves calls of
    different batch shapes back to back on one stream: no call may depend on
    what an earlier call (of another geometry and split count) left in it."""
    names = ["short_and_long_mix", "g8_long", "short_and_long_mix", "g16_tree_cut", "chain_cross_pages"]
    cases, outs, sizes = [], [], []
    for i, name in enumerate(names):
        parents, pre, Hq, Hkv, D = ATTN_CASES[name]
        cases.append(small_case(parents, pre, Hq=Hq, Hkv=Hkv, D=D, seed=40 + i))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    batches = [_batch(c, status) for c in cases]
    sizes = [jsv.jsv_tree_attention_workspace_size(b) for b, _ in batches]
    ws = torch.full((max(max(sizes), 256),), 0x5A, dtype=torch.uint8, device="cuda")
    keep = []
    for c, (b, dev) in zip(cases, batches):
        q, k, v = _dev_bf16(c["q"]), _dev_bf16(c["k_cache"]), _dev_bf16(c["v_cache"])
        T = int(c["node_offsets"][-1])
        out = torch.zeros((T, c["Hq"], c["D"]), dtype=torch.bfloat16, device="cuda")
        jsv.jsv_tree_attention(b, q, k, v, c["scale"], out, ws)
        keep.append((q, k, v, dev))
        outs.append(out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    from helpers import run_oracle_attention
    for name, c, out in zip(names, cases, outs):
        got = synth.bf16_bits_to_f32(_bits(out)).astype(np.float64)
        attention_close(got, run_oracle_attention(c), name)


# (64, 128, 40000): single CTAs with vocabulary units of 8 or 9 boxes, i.e.
# units that span two 128-row W tiles; (200, 128, 38500) and (256, 64, 38500):
# CTA pairs with more 256-row units than pairs, so the units left over are
# split into 16-node pieces
@pytest.mark.parametrize("T,d,V", [(1, 64, 1), (5, 128, 1000), (16, 256, 1024), (64, 512, 4099),
                                   (130, 192, 3000), (300, 1024, 20000), (200, 256, 2500), (256, 128, 257),
                                   (64, 128, 40000), (200, 128, 38500), (256, 64, 38500)])
def test_lmhead_argmax_shapes(T, d, V):
    rng = np.random.default_rng(T * 7 + V)
    H = bf16(rng.standard_normal((T, d)) / math.sqrt(d))
    W = bf16(rng.standard_normal((V, d)) / math.sqrt(d))
    a, t1, t2 = oracle.lmhead_top2(H, W)
    ok, _ = oracle.certify_margin(H, W, a, t1, t2)
    assert ok.mean() > 0.8
    arg = torch.empty(T, dtype=torch.int32, device="cuda")
    ml = torch.empty(T, dtype=torch.float32, device="cuda")
    ws = torch.zeros(jsv.jsv_lmhead_argmax_workspace_size(T, d, V), dtype=torch.uint8, device="cuda")
    jsv.jsv_lmhead_argmax(_dev_bf16(H), _dev_bf16(W), T, d, V, arg, ml, ws)
    torch.cuda.synchronize()
    g = arg.cpu().numpy()
    assert np.array_equal(g[ok], a[ok])
    assert np.all((g >= 0) & (g < V))
    assert np.allclose(ml.cpu().numpy()[ok], t1[ok], rtol=1e-4, atol=1e-5)


def test_lmhead_workspace_reused_without_clearing():
    """One workspace, zeroed once, serves back-to-back calls of different
    shapes on one stream with no synchronisation in between: every call must
    leave the keys and the completion counter zeroed for the next one."""
    shapes = [(64, 256, 5000), (16, 256, 5000), (64, 256, 5000), (100, 128, 3001), (3, 128, 3001)]
    ws = torch.zeros(jsv.jsv_lmhead_argmax_workspace_size(128, 256, 5000), dtype=torch.uint8, device="cuda")
    runs = []
    for i, (T, d, V) in enumerate(shapes):
        rng = np.random.default_rng(500 + i)
        H = bf16(rng.standard_normal((T, d)) / math.sqrt(d))
        W = bf16(rng.standard_normal((V, d)) / math.sqrt(d))
        arg = torch.empty(T, dtype=torch.int32, device="cuda")
        dh, dw = _dev_bf16(H), _dev_bf16(W)
        jsv.jsv_lmhead_argmax(dh, dw, T, d, V, arg, None, ws)
        runs.append((H, W, arg, dh, dw))
    torch.cuda.synchronize()
    for H, W, arg, _, _ in runs:
        a, t1, t2 = oracle.lmhead_top2(H, W)
        ok, _ = oracle.certify_margin(H, W, a, t1, t2)
        assert ok.mean() > 0.8
        assert np.array_equal(arg.cpu().numpy()[ok], a[ok])
    assert not ws.any().item()


def test_lmhead_ties_take_smallest_index():
    d, V, T = 64, 700, 3
    W = np.zeros((V, d), dtype=np.float32)
    W[[17, 300, 650]] = 1.0 / 8          # exact ties for every node
    H = np.full((T, d), 1.0 / 8, dtype=np.float32)
    arg = torch.empty(T, dtype=torch.int32, device="cuda")
    ws = torch.zeros(jsv.jsv_lmhead_argmax_workspace_size(T, d, V), dtype=torch.uint8, device="cuda")
    jsv.jsv_lmhead_argmax(_dev_bf16(bf16(H)), _dev_bf16(bf16(W)), T, d, V, arg, None, ws)
    torch.cuda.synchronize()
    assert arg.cpu().tolist() == [17, 17, 17]


def _walk_and_compact(parents, pre, tokens, argmax, max_path=None, fused=False, mutate=None):
    """The accept walk and the KV compaction, as two calls or as the fused
    jsv_accept_compact; `mutate` edits the case (to plant an input error)."""
    case = small_case(parents, pre, Hq=2, Hkv=2, D=64, seed=3)
    if mutate:
        mutate(case)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    batch, keep = _batch(case, status)
    B = len(parents)
    mp = max_path or max(len(p) for p in parents)
    path = torch.full((B, mp), 77, dtype=torch.int32, device="cuda")
    acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    bonus = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    nl = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    k, v = _dev_bf16(case["k_cache"]), _dev_bf16(case["v_cache"])
    if fused:
        jsv.jsv_accept_compact(batch, _dev_i32(tokens), _dev_i32(argmax), mp, path, acc, bonus, k, v, nl)
    else:
        jsv.jsv_accept_path(batch, _dev_i32(tokens), _dev_i32(argmax), mp, path, acc, bonus)
        jsv.jsv_kv_compact(batch, k, v, path, mp, acc, nl)
    torch.cuda.synchronize()
    return case, dict(path=path.cpu().numpy(), acc=acc.cpu().numpy(), bonus=bonus.cpu().numpy(),
                      new_len=nl.cpu().numpy(), k=_bits(k), v=_bits(v), status=int(status.item()))


@pytest.mark.parametrize("fused", [False, True])
def test_walk_and_compaction_random_batches(fused):
    rng = np.random.default_rng(9)
    for trial in range(6):
        B = int(rng.integers(1, 9))
        parents = [synth.tiny_tree(rng, int(rng.integers(1, 200)), 40, 3) for _ in range(B)]
        pre = [int(rng.integers(0, 100)) for _ in range(B)]
        T = sum(len(p) for p in parents)
        argmax = rng.integers(0, 6, T)        # small vocab: duplicates and long paths
        tokens = rng.integers(0, 6, T)
        offs = np.concatenate([[0], np.cumsum([len(p) for p in parents])])
        for b, p in enumerate(parents):
            for c in range(1, len(p)):
                if rng.random() < 0.8:
                    tokens[offs[b] + c] = argmax[offs[b] + p[c]]
        case, got = _walk_and_compact(parents, pre, tokens, argmax, fused=fused)
        assert got["status"] == 0
        ref = oracle.accept_batch(offs, np.concatenate(parents), tokens, argmax)
        kref, vref = case["k_cache"].copy(), case["v_cache"].copy()
        nl = oracle.kv_compact(kref, vref, case["page_table"], case["prefix_len"], [r[0] for r in ref])
        for b, (p, a, bo) in enumerate(ref):
            assert got["acc"][b] == a and got["bonus"][b] == bo
            assert got["path"][b, :a + 1].tolist() == p
        assert np.array_equal(got["new_len"], nl)
        assert np.array_equal(got["k"], kref) and np.array_equal(got["v"], vref)


@pytest.mark.parametrize("fused", [False, True])
def test_full_depth_chain_and_zero_accept(fused):
    n = 300
    chain = np.arange(-1, n - 1)
    argmax = np.arange(n) + 1000
    tokens = np.concatenate([[5], argmax[:-1]])                 # everything matches
    case, got = _walk_and_compact([chain, np.array([-1, 0, 0])], [33, 7],
                                  np.concatenate([tokens, [1, 2, 3]]),
                                  np.concatenate([argmax, [9, 9, 9]]), fused=fused)
    assert got["status"] == 0
    assert got["acc"].tolist() == [n - 1, 0]
    assert got["path"][0].tolist() == list(range(n))
    assert got["new_len"].tolist() == [33 + n, 8]


@pytest.mark.parametrize("fused", [False, True])
def test_path_longer_than_max_path_is_reported(fused):
    n = 10
    chain = np.arange(-1, n - 1)
    argmax = np.arange(n) + 50
    tokens = np.concatenate([[0], argmax[:-1]])
    case, got = _walk_and_compact([chain], [3], tokens, argmax, max_path=4, fused=fused)
    assert got["status"] == jsv.JSV_ERR_DEVICE_INPUT
    assert got["path"][0].tolist() == [0, 1, 2, 3]


def _bad_parent(case):
    case["parent"] = case["parent"].copy()
    case["parent"][2] = 5                      # parent index above the node's own


def _bad_tree_page(case):
    case["page_table"] = case["page_table"].copy()
    case["page_table"][0, case["prefix_len"][0] // 16] = case["num_pages"] + 3


@pytest.mark.parametrize("mutate,max_path", [(None, 4), (_bad_parent, None), (_bad_tree_page, None)])
def test_fused_accept_compact_equals_the_two_calls(mutate, max_path):
    """Bit-for-bit the same outputs and status as jsv_accept_path +
    jsv_kv_compact, on a good batch cut by max_path and on inputs that the
    device rejects (a malformed parent array, an unmapped tree page)."""
    rng = np.random.default_rng(21)
    parents = [synth.tiny_tree(rng, 30, 8, 2), np.arange(-1, 12), synth.tiny_tree(rng, 50, 10, 3)]
    pre = [37, 16, 5]
    T = sum(len(p) for p in parents)
    argmax = rng.integers(0, 4, T)
    tokens = rng.integers(0, 4, T)
    offs = np.concatenate([[0], np.cumsum([len(p) for p in parents])])
    for b, p in enumerate(parents):
        for c in range(1, len(p)):
            if rng.random() < 0.85:
                tokens[offs[b] + c] = argmax[offs[b] + p[c]]
    _, two = _walk_and_compact(parents, pre, tokens, argmax, max_path=max_path, mutate=mutate)
    _, one = _walk_and_compact(parents, pre, tokens, argmax, max_path=max_path, mutate=mutate, fused=True)
    assert two["status"] == jsv.JSV_ERR_DEVICE_INPUT
    for key in two:
        assert np.array_equal(np.asarray(one[key]), np.asarray(two[key])), key


def test_malformed_parent_is_reported_not_trapped():
    case = small_case([np.array([-1, 0, 1, 1])], [20], Hq=2, Hkv=1, D=64, seed=4)
    case["parent"] = np.array([-1, 0, 3, 1], dtype=np.int32)    # parent[2] = 3 > 2
    out, st = run_attention(case)
    assert st == jsv.JSV_ERR_DEVICE_INPUT


def test_page_out_of_range_is_reported():
    case = small_case([np.array([-1, 0])], [40], Hq=2, Hkv=1, D=64, seed=5)
    case["page_table"] = case["page_table"].copy()
    case["page_table"][0, 1] = case["num_pages"] + 5
    out, st = run_attention(case)
    assert st == jsv.JSV_ERR_DEVICE_INPUT


# Chains whose row counts straddle the 64-, 128- and 256-row boundaries of the
# CTA's row groups and warps, with one and several key tiles: each warp of a
# group may run a tile ahead of the others, and every row must still see the
# P of its own tile.
@pytest.mark.parametrize("n,pre", [(30, 29), (33, 29), (41, 29), (64, 29), (64, 200), (41, 300)])
def test_attention_row_groups_and_tiles(n, pre):
    case = small_case([np.arange(-1, n - 1)], [pre], Hq=8, Hkv=2, D=128, seed=11)
    got, st = run_attention(case)
    assert st == 0
    attention_close(got, dense_tree_attention(case), f"chain n={n} prefix={pre}")
