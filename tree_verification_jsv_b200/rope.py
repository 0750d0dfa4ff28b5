"""Rotary position tables for the tree Q/K/V projection call.

``rope_tables(theta, D, max_pos)`` returns fp32 cos and sin tables of shape
[max_pos][D/2] with angle p * theta^(-2i/D) (computed in float64, then
rounded); rows are positions, columns the rotation pairs (i, i + D/2) of the
rotate-half convention.  Callers pass these tables to jsv_tree_qkv_rope.
"""
from __future__ import annotations

import numpy as np


def rope_tables(theta: float, D: int, max_pos: int):
    inv = theta ** (-np.arange(0, D // 2, dtype=np.float64) * 2.0 / D)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
