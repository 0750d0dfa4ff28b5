"""Pins for the tree Q/K/V projection + rotary oracle."""
import math

import numpy as np

import oracle
from helpers import bf16, small_case
from tree_verification_jsv_b200 import rope, synth


def test_rotation_matches_complex_multiplication_and_preserves_norm():
    rng = np.random.default_rng(0)
    D = 16
    cos, sin = rope.rope_tables(10000.0, D, 50)
    for pos in (0, 1, 7, 49):
        x = rng.standard_normal(D)
        y = oracle.rope_rotate(x, cos[pos].astype(np.float64), sin[pos].astype(np.float64))
        z = (x[:D // 2] + 1j * x[D // 2:]) * (cos[pos] + 1j * sin[pos])      # complex form
        assert np.allclose(y, np.concatenate([z.real, z.imag]), atol=1e-12)
        assert abs(np.linalg.norm(y) - np.linalg.norm(x)) < 1e-6 * np.linalg.norm(x)
    assert np.array_equal(oracle.rope_rotate(np.arange(D, dtype=float), cos[0].astype(float),
                                             sin[0].astype(float)), np.arange(D, dtype=float))


def test_relative_position_property():
    # <R(p) q, R(p') k> depends only on p - p'
    rng = np.random.default_rng(1)
    D = 32
    cos, sin = rope.rope_tables(1e6, D, 200)
    c64, s64 = cos.astype(np.float64), sin.astype(np.float64)
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    dots = [oracle.rope_rotate(q, c64[p + 5], s64[p + 5]) @ oracle.rope_rotate(k, c64[p], s64[p])
            for p in (0, 17, 90, 150)]
    assert np.allclose(dots, dots[0], rtol=1e-5, atol=1e-6)


def test_projection_positions_and_cache_slots():
    rng = np.random.default_rng(2)
    Hq, Hkv, D, d = 4, 2, 16, 32
    parents = [np.array([-1, 0, 0, 1, 3]), np.array([-1, 0])]
    case = small_case(parents, [19, 3], Hq=Hq, Hkv=Hkv, D=D, seed=3)
    T = 7
    x = bf16(rng.standard_normal((T, d)) / math.sqrt(d))
    w = bf16(rng.standard_normal(((Hq + 2 * Hkv) * D, d)) / math.sqrt(d))
    cos, sin = rope.rope_tables(1e6, D, 64)
    kc0, vc0 = case["k_cache"].copy(), case["v_cache"].copy()
    kc, vc = kc0.copy(), vc0.copy()
    q, kk, vv = oracle.tree_qkv_rope(x=x, w_qkv=w, Hq=Hq, Hkv=Hkv, D=D, page_table=case["page_table"],
                                     prefix_len=case["prefix_len"], node_offsets=case["node_offsets"],
                                     parent=case["parent"], rope_cos=cos, rope_sin=sin, k_cache=kc, v_cache=vc)
    Y = synth.bf16_bits_to_f32(x).astype(np.float64) @ synth.bf16_bits_to_f32(w).astype(np.float64).T
    # node 4 of request 0 is at depth 3 -> position 19 + 3; its V is unrotated, K rotated there
    pos = 22
    assert np.allclose(vv[4, 1], Y[4, (Hq + Hkv + 1) * D:(Hq + Hkv + 2) * D])
    assert np.allclose(kk[4, 0], oracle.rope_rotate(Y[4, Hq * D:(Hq + 1) * D], cos[pos].astype(float),
                                                    sin[pos].astype(float)))
    assert np.allclose(q[4, 3], oracle.rope_rotate(Y[4, 3 * D:4 * D], cos[pos].astype(float), sin[pos].astype(float)))
    # request 1's root (node 5) at position 3, written to slot 3; nothing else changes
    changed = [(b, s) for b, P, n in [(0, 19, 5), (1, 3, 2)] for s in range(P, P + n)]
    flat_k0, flat_k = kc0.reshape(-1, Hkv, D), kc.reshape(-1, Hkv, D)
    rows = set()
    for b, s in changed:
        rows.add(int(case["page_table"][b, s // 16]) * 16 + s % 16)
    untouched = [r for r in range(flat_k0.shape[0]) if r not in rows]
    assert np.array_equal(flat_k0[untouched], flat_k[untouched])
    assert np.array_equal(vc0.reshape(-1, Hkv, D)[untouched], vc.reshape(-1, Hkv, D)[untouched])
    r5 = int(case["page_table"][1, 0]) * 16 + 3
    assert np.array_equal(flat_k[r5, 1], oracle._f64_to_bf16_bits(kk[5, 1]))
