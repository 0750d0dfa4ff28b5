"""Properties of the seeded workload generator (shapes, trees, paging)."""
import numpy as np
import pytest

from tree_verification_jsv_b200 import synth


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 1e-3, 0.0], dtype=np.float32)
    b = synth.f32_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(b)
    assert back[0] == 1.0
    assert back[1] == 1.0                       # tie rounds to even (down)
    assert back[2] == 1.0 + 2 ** -7             # tie rounds to even (up)
    assert back[3] == -2.5 and back[5] == 0.0
    assert abs(back[4] - 1e-3) <= 1e-3 * 2 ** -8


def test_draws_do_not_depend_on_blocking():
    a = synth.normal_bf16(5, "q", 10_000, 0.5)
    b = synth.normal_bf16(5, "q", 10_000, 0.5)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, synth.normal_bf16(6, "q", 10_000, 0.5))


@pytest.mark.parametrize("budget,depth,k", [(64, 8, 4), (256, 16, 8), (512, 16, 8), (40, 12, 4)])
def test_budget_tree_shape(budget, depth, k):
    p = synth.budget_tree(np.random.default_rng(1), budget, depth, k)
    assert len(p) == budget and p[0] == -1
    assert all(0 <= p[i] < i for i in range(1, budget))
    d = synth.depths(p)
    assert d.max() == depth                      # the spine realises the depth
    assert np.all(np.diff(d) >= 0)               # BFS order
    counts = np.bincount(p[1:], minlength=budget)
    assert counts.max() <= k


def test_tiny_tree_limits():
    p = synth.tiny_tree(np.random.default_rng(2), 16, 5, 3)
    assert synth.depths(p).max() <= 5
    assert np.bincount(p[1:]).max() <= 3


@pytest.mark.parametrize("name", list(synth.SHAPES))
def test_workload_geometry(name):
    wl = synth.make_workload(name, values=False, lmhead=False)
    B, Hq, Hkv, D, d, V = synth.SHAPES[name]
    assert wl.B == B and len(wl.prefix_len) == B
    mapped = wl.page_table[wl.page_table >= 0]
    assert len(np.unique(mapped)) == len(mapped)          # no page shared
    assert mapped.max() < wl.num_pages
    for b in range(B):
        need = (wl.prefix_len[b] + wl.node_offsets[b + 1] - wl.node_offsets[b] + 15) // 16
        assert np.all(wl.page_table[b, :need] >= 0)
        sl = wl.request_nodes(b)
        assert wl.parent[sl.start] == -1 and not wl.tok_flag[sl.start]
    if name == "ragged16":
        assert wl.prefix_len.min() >= 512 and wl.prefix_len.max() <= 8192
        n = np.diff(wl.node_offsets)
        assert n.min() >= 32 and n.max() <= 128
    if name == "30b_512x4":
        assert np.all(wl.prefix_len == 32768) and np.all(np.diff(wl.node_offsets) == 512)


def test_plant_tokens_follows_flags():
    wl = synth.make_workload("tiny", values=False, lmhead=False)
    argmax = np.arange(wl.T) + 500
    tok = synth.plant_tokens(wl, argmax)
    for t in range(wl.T):
        if wl.tok_flag[t]:
            assert tok[t] == argmax[wl.parent[t]]      # tiny: one request, base 0
        else:
            assert tok[t] == wl.tok_uniform[t]
