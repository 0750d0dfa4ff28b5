"""GPU parity of the whole verify step against the oracle, on every named
workload at full size, through the C ABI.

Bit-exact: argmax (certified goldens), accepted path, accept length, bonus,
new lengths and the ENTIRE K and V cache buffers after compaction.
Attention: within the tolerance in ``helpers.attention_close`` on all rows
(small workloads) or on a seeded sample of rows the oracle computes one by
one (large workloads).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import attention_close, golden_workload

pytestmark = pytest.mark.gpu

WORKLOADS = ["tiny", "8b_64", "8b_256", "ragged16", "30b_512x4"]


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _sample_rows(wl, n, seed):
    """Seeded rows plus the deepest node of every request and every root."""
    rng = np.random.default_rng(seed)
    rows = set()
    for b in range(wl.B):
        sl = wl.request_nodes(b)
        from tree_verification_jsv_b200 import synth
        dep = synth.depths(wl.parent[sl])
        for t in (sl.start, sl.start + int(np.argmax(dep))):
            rows.add((t, 0))
            rows.add((t, wl.Hq - 1))
    while len(rows) < n:
        rows.add((int(rng.integers(wl.T)), int(rng.integers(wl.Hq))))
    return np.array(sorted(rows), dtype=np.int32)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_jsv_b200 import build, jsv
    build.build()
    jsv.load()


@pytest.mark.parametrize("name", WORKLOADS)
def test_verify_step_matches_oracle(name):
    from tree_verification_jsv_b200.step import VerifyStep
    wl, tokens, gold_arg = golden_workload(name)
    k0, v0 = wl.k_cache.copy(), wl.v_cache.copy()
    st = VerifyStep(wl, tokens)
    st.run()
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0

    # LM head argmax: bit-exact against the certified fp64 oracle
    arg = st.argmax.cpu().numpy()
    assert np.array_equal(arg, gold_arg), f"{(arg != gold_arg).sum()} argmax mismatches"

    # walk
    ref = oracle.accept_batch(wl.node_offsets, wl.parent, tokens, gold_arg)
    path = st.path.cpu().numpy()
    acc = st.accept_len.cpu().numpy()
    bonus = st.bonus.cpu().numpy()
    for b, (p, a, bo) in enumerate(ref):
        assert acc[b] == a and bonus[b] == bo
        assert path[b, :a + 1].tolist() == p
        assert np.all(path[b, a + 1:] == -1)

    # compaction: whole buffers, bytewise
    kref, vref = k0.copy(), v0.copy()
    new_len = oracle.kv_compact(kref, vref, wl.page_table, wl.prefix_len, [r[0] for r in ref])
    assert np.array_equal(st.new_len.cpu().numpy(), new_len)
    assert np.array_equal(_bits(st.k_cache), kref)
    assert np.array_equal(_bits(st.v_cache), vref)

    # attention (computed before compaction, on the original cache)
    out = _bits(st.out)
    wl.k_cache, wl.v_cache = k0, v0
    from tree_verification_jsv_b200 import synth
    got_all = synth.bf16_bits_to_f32(out).astype(np.float64)
    if wl.T * wl.Hq <= 4096:
        want = oracle.tree_attention_wl(wl)
        attention_close(got_all, want, name)
    else:
        rows = _sample_rows(wl, 384, seed=7)
        want = oracle.tree_attention_wl(wl, rows=rows)
        attention_close(got_all[rows[:, 0], rows[:, 1]], want, name)
