"""Pins for the LM-head argmax oracle (temperature-0 greedy choice of the
target's own logits; JetSpec README, "JetSpec / Overview" and the
temperature=0.0 sampling parameters of its examples)."""
from fractions import Fraction

import numpy as np

import oracle
from helpers import bf16
from tree_verification_jsv_b200 import synth


def _exact_argmax(H, W):
    """Brute force in exact rational arithmetic: the smallest v attaining the max."""
    Hf = [[Fraction(float(x)) for x in row] for row in synth.bf16_bits_to_f32(H)]
    Wf = [[Fraction(float(x)) for x in row] for row in synth.bf16_bits_to_f32(W)]
    out, top = [], []
    for h in Hf:
        best, arg = None, -1
        for v, w in enumerate(Wf):
            s = sum(a * b for a, b in zip(h, w))
            if best is None or s > best:
                best, arg = s, v
        out.append(arg)
        top.append(best)
    return np.array(out), top


def test_matches_exact_rational_brute_force():
    rng = np.random.default_rng(0)
    H = bf16(rng.standard_normal((6, 12)) / 3)
    W = bf16(rng.standard_normal((41, 12)) / 3)
    arg, top1, _ = oracle.lmhead_top2(H, W, chunk=8)     # several chunks + a ragged tail
    want, top = _exact_argmax(H, W)
    assert np.array_equal(arg, want)
    assert np.allclose(top1, [float(t) for t in top], rtol=0, atol=1e-15)


def test_ties_take_smallest_index_within_and_across_chunks():
    # small integers: every logit is exact in fp64, so ties are real ties
    H = bf16(np.array([[1, 2, 0, 1], [0, 1, 1, 0]], dtype=np.float32))
    W = np.zeros((20, 4), dtype=np.float32)
    W[3] = [1, 1, 0, 0]      # row 0: 3, row 1: 1
    W[5] = [1, 1, 0, 0]      # duplicate of 3 inside the same chunk
    W[9] = [1, 1, 0, 0]      # duplicate in a later chunk
    W[12] = [0, 0, 1, 1]     # row 1: 1  (ties with 3,5,9 for row 1)
    W[17] = [0, 1, 1, 0]     # row 1: 2 (unique max for row 1)
    arg, top1, top2 = oracle.lmhead_top2(H, bf16(W), chunk=8)
    assert list(arg) == [3, 17]
    assert top1[0] == 3 and top2[0] == 3                 # tie: zero margin
    assert top1[1] == 2 and top2[1] == 1


def test_runner_up_matches_sorted_logits():
    rng = np.random.default_rng(1)
    H = bf16(rng.standard_normal((5, 16)))
    W = bf16(rng.standard_normal((300, 16)))
    arg, t1, t2 = oracle.lmhead_top2(H, W, chunk=64)
    L = synth.bf16_bits_to_f32(H).astype(np.float64) @ synth.bf16_bits_to_f32(W).astype(np.float64).T
    srt = np.sort(L, axis=1)
    assert np.allclose(t1, srt[:, -1], atol=1e-14)
    assert np.allclose(t2, srt[:, -2], atol=1e-14)


def test_one_hot_rows_pick_the_planted_index():
    d, V = 32, 100
    W = np.zeros((V, d), dtype=np.float32)
    for v in range(V):
        W[v, v % d] = 1.0 + v / 1000.0
    H = np.zeros((4, d), dtype=np.float32)
    for i, j in enumerate([0, 7, 31, 5]):
        H[i, j] = 1.0
    arg = oracle.lmhead_argmax(bf16(H), bf16(W))
    # column j is hit by v = j, j+32, j+64, j+96 (if < V); the largest weight wins
    want = [max(v for v in range(V) if v % d == j) for j in [0, 7, 31, 5]]
    Wb = synth.bf16_bits_to_f32(bf16(W))
    assert list(arg) == [int(np.argmax(Wb[:, j])) for j in [0, 7, 31, 5]]
    assert len(want) == 4


def test_certification_bound_is_sound_against_fp32_orders():
    """Certified rows keep their argmax under several fp32 summation orders
    (forward, reversed, pairwise, blocked by 16), the way a kernel might add."""
    rng = np.random.default_rng(2)
    d, V, T = 256, 512, 64
    H = bf16(rng.standard_normal((T, d)) / np.sqrt(d))
    W = bf16(rng.standard_normal((V, d)) / np.sqrt(d))
    arg, t1, t2 = oracle.lmhead_top2(H, W)
    ok, ratio = oracle.certify_margin(H, W, arg, t1, t2)
    Hf = synth.bf16_bits_to_f32(H)
    Wf = synth.bf16_bits_to_f32(W)
    prod = (Hf[:, None, :] * Wf[None, :, :]).astype(np.float32)     # exact products
    def fwd(p):
        acc = np.zeros(p.shape[:2], np.float32)
        for k in range(p.shape[2]):
            acc = (acc + p[:, :, k]).astype(np.float32)
        return acc
    orders = [fwd(prod), fwd(prod[:, :, ::-1]),
              fwd(np.stack([fwd(prod[:, :, k:k + 16]) for k in range(0, d, 16)], axis=2))]
    assert ok.sum() > T // 2
    for L in orders:
        assert np.array_equal(np.argmax(L, axis=1)[ok], arg[ok])


def test_certification_rejects_exact_ties_and_tiny_gaps():
    H = bf16(np.array([[1, 0], [1, 0]], dtype=np.float32))
    W = bf16(np.array([[1, 0], [1, 0], [0.5, 0]], dtype=np.float32))
    arg, t1, t2 = oracle.lmhead_top2(H, W)
    ok, ratio = oracle.certify_margin(H, W, arg, t1, t2)
    assert list(arg) == [0, 0] and not ok.any() and np.all(ratio == 0)
