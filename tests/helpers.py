"""Small seeded cases for oracle pins and GPU parity (test-side only)."""
import math

import numpy as np

from tree_verification_jsv_b200 import synth


def bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f64(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def small_case(parents, prefixes, Hq=4, Hkv=2, D=16, seed=0, identity=False, q_scale=1.0):
    """Arbitrary trees (request-local parent arrays) over paged caches with
    N(0,1)/sqrt(D) bf16 values drawn from a seeded generator."""
    rng = np.random.default_rng(seed)
    nodes = [len(p) for p in parents]
    offs = np.zeros(len(parents) + 1, dtype=np.int32)
    offs[1:] = np.cumsum(nodes)
    table, num_pages = synth.make_paging(seed, prefixes, nodes, identity=identity)
    T = int(offs[-1])
    s = 1.0 / math.sqrt(D)
    return dict(
        Hq=Hq, Hkv=Hkv, D=D,
        page_table=table, num_pages=num_pages,
        prefix_len=np.asarray(prefixes, dtype=np.int32),
        node_offsets=offs,
        parent=np.concatenate([np.asarray(p, dtype=np.int32) for p in parents]),
        q=bf16(rng.standard_normal((T, Hq, D)) * s * q_scale),
        k_cache=bf16(rng.standard_normal((num_pages, 16, Hkv, D)) * s),
        v_cache=bf16(rng.standard_normal((num_pages, 16, Hkv, D)) * s),
        scale=float(np.float32(1.0 / math.sqrt(D))),
    )


def logical_rows(cache_bits, page_table, b, n_slots):
    """[n_slots, Hkv, D] fp64 rows of request b's logical sequence."""
    flat = cache_bits.reshape(-1, cache_bits.shape[2], cache_bits.shape[3])
    s = np.arange(n_slots)
    phys = page_table[b, s // 16].astype(np.int64) * 16 + s % 16
    return f64(flat[phys])


def ancestor_matrix(parent):
    """A[i, j] = True iff j is i or an ancestor of i (topological input)."""
    n = len(parent)
    A = np.zeros((n, n), dtype=bool)
    for i in range(n):
        if parent[i] >= 0:
            A[i] = A[parent[i]]
        A[i, i] = True
    return A


def dense_tree_attention(case):
    """Independent reference: numpy dense attention over each request's
    logical sequence with an explicit [N, P+N] visibility mask."""
    Hq, Hkv, D = case["Hq"], case["Hkv"], case["D"]
    G = Hq // Hkv
    offs = case["node_offsets"]
    out = np.zeros((int(offs[-1]), Hq, D))
    for b in range(len(offs) - 1):
        s0, s1 = int(offs[b]), int(offs[b + 1])
        n = s1 - s0
        P = int(case["prefix_len"][b])
        K = logical_rows(case["k_cache"], case["page_table"], b, P + n)
        V = logical_rows(case["v_cache"], case["page_table"], b, P + n)
        mask = np.zeros((n, P + n), dtype=bool)
        mask[:, :P] = True
        mask[:, P:] = ancestor_matrix(case["parent"][s0:s1])
        for h in range(Hq):
            g = h // G
            Q = f64(case["q"][s0:s1, h])
            S = case["scale"] * (Q @ K[:, g].T)
            S[~mask] = -np.inf
            S -= S.max(axis=1, keepdims=True)
            Pm = np.exp(S)
            Pm /= Pm.sum(axis=1, keepdims=True)
            out[s0:s1, h] = Pm @ V[:, g]
    return out


def run_oracle_attention(case, rows=None):
    import oracle
    return oracle.tree_attention(Hq=case["Hq"], Hkv=case["Hkv"], D=case["D"],
                                 page_table=case["page_table"], prefix_len=case["prefix_len"],
                                 node_offsets=case["node_offsets"], parent=case["parent"],
                                 q=case["q"], k_cache=case["k_cache"], v_cache=case["v_cache"],
                                 scale=case["scale"], rows=rows)


def golden(name):
    import json
    from pathlib import Path
    return json.loads((Path(__file__).resolve().parent / "golden" / f"lmhead_{name}.json").read_text())


def golden_workload(name, **kw):
    """Workload with the certified hidden-row redraws and planted tokens."""
    g = golden(name)
    wl = synth.make_workload(name, redraws={int(k): v for k, v in g["redraws"].items()}, **kw)
    tokens = np.asarray(g["tokens"], dtype=np.int32)
    return wl, tokens, np.asarray(g["argmax"], dtype=np.int64)


def attention_close(got, want, what=""):
    """Tolerance: |g - o| <= 2e-2 + 1e-2 |o| elementwise (bf16 output, fp32
    accumulation), plus a tight check |g - o| <= 1e-2 |o| + 1e-2 max|o| so a
    near-zero or partial result cannot hide inside the absolute term.

    The second term of the tight check is relative to the tensor's largest
    output, not to each element: the tensor-core PV product takes the softmax
    weights in bf16 (its operand type), and that rounding (up to 2^-9 of each
    weight) leaves an error that scales with the value rows, so an output that
    is small only because its weighted values cancel carries a larger
    relative error."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    assert np.all(err <= 2e-2 + 1e-2 * np.abs(want)), f"{what}: max abs err {err.max()}"
    tight = 1e-2 * np.abs(want) + 1e-2 * np.abs(want).max()
    bad = err > tight
    assert not bad.any(), (f"{what}: {bad.sum()} elems beyond tight bound, max err {err.max()}, "
                           f"max|o| {np.abs(want).max()}")
    return float(err.max())


def _bits_t(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def sample_rows(wl, n, seed):
    """Seeded (node, head) rows plus the root and the deepest node of every
    request (first and last head)."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(wl.B):
        sl = wl.request_nodes(b)
        dep = synth.depths(wl.parent[sl])
        for t in (sl.start, sl.start + int(np.argmax(dep))):
            rows.add((t, 0))
            rows.add((t, wl.Hq - 1))
    while len(rows) < n:
        rows.add((int(rng.integers(wl.T)), int(rng.integers(wl.Hq))))
    return np.array(sorted(rows), dtype=np.int32)


def assert_step_matches_oracle(st, wl, tokens, gold_arg, k0, v0, what):
    """Every output of one verify step held by ``st`` (a VerifyStep that ran
    once on caches k0/v0) against the oracle: argmax bit-exact against the
    certified goldens, path / accept length / bonus / new length bit-exact,
    the ENTIRE K and V caches bytewise, and the attention within the
    tolerance of ``attention_close`` (all rows of small workloads, a seeded
    sample of rows computed one by one on large ones)."""
    import oracle
    assert int(st.status.item()) == 0, what
    arg = st.argmax.cpu().numpy()
    assert np.array_equal(arg, gold_arg), f"{what}: {(arg != gold_arg).sum()} argmax mismatches"
    ref = oracle.accept_batch(wl.node_offsets, wl.parent, tokens, gold_arg)
    path = st.path.cpu().numpy()
    acc = st.accept_len.cpu().numpy()
    bonus = st.bonus.cpu().numpy()
    for b, (p, a, bo) in enumerate(ref):
        assert acc[b] == a and bonus[b] == bo, what
        assert path[b, :a + 1].tolist() == p, what
        assert np.all(path[b, a + 1:] == -1), what
    kref, vref = k0.copy(), v0.copy()
    new_len = oracle.kv_compact(kref, vref, wl.page_table, wl.prefix_len, [r[0] for r in ref])
    assert np.array_equal(st.new_len.cpu().numpy(), new_len), what
    assert np.array_equal(_bits_t(st.k_cache), kref), what
    assert np.array_equal(_bits_t(st.v_cache), vref), what
    # attention (computed before the compaction, on the original caches)
    saved = wl.k_cache, wl.v_cache
    wl.k_cache, wl.v_cache = k0, v0
    try:
        got_all = synth.bf16_bits_to_f32(_bits_t(st.out)).astype(np.float64)
        if wl.T * wl.Hq <= 4096:
            attention_close(got_all, oracle.tree_attention_wl(wl), what)
        else:
            rows = sample_rows(wl, 384, seed=7)
            want = oracle.tree_attention_wl(wl, rows=rows)
            attention_close(got_all[rows[:, 0], rows[:, 1]], want, what)
    finally:
        wl.k_cache, wl.v_cache = saved
