"""GPU parity of the tree Q/K/V projection + rotary + paged K/V append with
its oracle: q and the written K/V within the bf16 tolerance, every other
cache byte unchanged."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import attention_close, bf16, small_case
from tree_verification_jsv_b200 import jsv, rope, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from tree_verification_jsv_b200 import build
    build.build()
    jsv.load()


def _dev_i32(a):
    return torch.as_tensor(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


CASES = {
    "small_d64": ([synth.tiny_tree(np.random.default_rng(1), 13, 5, 3), np.array([-1, 0, 1])], [21, 0],
                  4, 2, 64, 128),
    "qwen3_8b_64": ([synth.budget_tree(np.random.default_rng(2), 64, 8, 4)], [2048], 32, 8, 128, 4096),
    "ragged_300": ([synth.budget_tree(np.random.default_rng(3), n, 10, 4) for n in (100, 37, 163)],
                   [500, 1700, 33], 32, 8, 128, 1024),
    "g8_d2048": ([synth.budget_tree(np.random.default_rng(4), 96, 12, 8)], [777], 32, 4, 128, 2048),
    # K splits of 4 (24 head tiles) and of 2 (64 head tiles), with node counts
    # that leave a partial 32-node slice
    "ksplit4_40_nodes": ([synth.budget_tree(np.random.default_rng(5), 40, 6, 4)], [300], 16, 4, 128, 1024),
    "ksplit2_two_requests": ([synth.tiny_tree(np.random.default_rng(6), 29, 6, 3),
                              synth.tiny_tree(np.random.default_rng(7), 21, 5, 3)], [90, 17], 48, 8, 128, 512),
    # one 256-node tree of Qwen3-8B shapes: a K split of 2 whose eight 32-node
    # slices pass through the first CTA's slots (handshake phases wrap)
    "qwen3_8b_256": ([synth.budget_tree(np.random.default_rng(9), 256, 16, 8)], [4000], 32, 8, 128, 4096),
}


@pytest.mark.parametrize("name", list(CASES))
def test_matches_oracle(name):
    parents, pre, Hq, Hkv, D, d = CASES[name]
    case = small_case(parents, pre, Hq=Hq, Hkv=Hkv, D=D, seed=5)
    T = int(case["node_offsets"][-1])
    rng = np.random.default_rng(6)
    x = bf16(rng.standard_normal((T, d)) / math.sqrt(d))
    w = bf16(rng.standard_normal(((Hq + 2 * Hkv) * D, d)) / math.sqrt(d))
    max_pos = max(pre) + 64
    cos, sin = rope.rope_tables(1e6, D, max_pos)
    kc0, vc0 = case["k_cache"].copy(), case["v_cache"].copy()

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    offs = case["node_offsets"]
    keep = [_dev_i32(case["page_table"]), _dev_i32(case["prefix_len"]), _dev_i32(offs), _dev_i32(case["parent"])]
    batch = jsv.make_batch(B=len(parents), Hq=Hq, Hkv=Hkv, D=D, max_pages_per_req=case["page_table"].shape[1],
                           num_pages=case["num_pages"], total_nodes=T, max_nodes=int(np.diff(offs).max()),
                           max_prefix=max(pre), page_table=keep[0], prefix_len=keep[1], node_offsets=keep[2],
                           parent=keep[3], dev_status=status)
    q = torch.zeros((T, Hq, D), dtype=torch.bfloat16, device="cuda")
    k, v = _dev_bf16(kc0), _dev_bf16(vc0)
    jsv.jsv_tree_qkv_rope(batch, _dev_bf16(x), _dev_bf16(w), d, torch.as_tensor(cos).cuda(),
                          torch.as_tensor(sin).cuda(), max_pos, q, k, v)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    kr, vr = kc0.copy(), vc0.copy()
    qref, kref, vref = oracle.tree_qkv_rope(x=x, w_qkv=w, Hq=Hq, Hkv=Hkv, D=D, page_table=case["page_table"],
                                            prefix_len=case["prefix_len"], node_offsets=offs,
                                            parent=case["parent"], rope_cos=cos, rope_sin=sin,
                                            k_cache=kr, v_cache=vr)
    attention_close(synth.bf16_bits_to_f32(_bits(q)).astype(np.float64), qref, f"{name} q")
    kg, vg = _bits(k), _bits(v)
    # written slots: compare values; all other bytes: identical
    flat = lambda c: c.reshape(-1, Hkv, D)
    written = []
    for b in range(len(parents)):
        for i in range(int(offs[b + 1] - offs[b])):
            s = pre[b] + i
            written.append(int(case["page_table"][b, s // 16]) * 16 + s % 16)
    mask = np.ones(flat(kg).shape[0], dtype=bool)
    mask[written] = False
    assert np.array_equal(flat(kg)[mask], flat(kc0)[mask]) and np.array_equal(flat(vg)[mask], flat(vc0)[mask])
    tk = np.stack([synth.bf16_bits_to_f32(flat(kg)[r]) for r in written]).astype(np.float64)
    tv = np.stack([synth.bf16_bits_to_f32(flat(vg)[r]) for r in written]).astype(np.float64)
    attention_close(tk, kref, f"{name} k")
    attention_close(tv, vref, f"{name} v")


def test_position_past_table_is_reported():
    case = small_case([np.array([-1, 0, 1])], [30], Hq=2, Hkv=1, D=64, seed=7)
    T, d = 3, 64
    rng = np.random.default_rng(8)
    x, w = bf16(rng.standard_normal((T, d)) * 0.1), bf16(rng.standard_normal((4 * 64, d)) * 0.1)
    cos, sin = rope.rope_tables(1e4, 64, 31)          # positions 30, 31, 32 -> only 30 fits
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    keep = [_dev_i32(case["page_table"]), _dev_i32(case["prefix_len"]), _dev_i32(case["node_offsets"]),
            _dev_i32(case["parent"])]
    batch = jsv.make_batch(B=1, Hq=2, Hkv=1, D=64, max_pages_per_req=case["page_table"].shape[1],
                           num_pages=case["num_pages"], total_nodes=T, max_nodes=3, max_prefix=30,
                           page_table=keep[0], prefix_len=keep[1], node_offsets=keep[2], parent=keep[3],
                           dev_status=status)
    q = torch.zeros((T, 2, 64), dtype=torch.bfloat16, device="cuda")
    jsv.jsv_tree_qkv_rope(batch, _dev_bf16(x), _dev_bf16(w), d, torch.as_tensor(cos).cuda(),
                          torch.as_tensor(sin).cuda(), 31, q, _dev_bf16(case["k_cache"]), _dev_bf16(case["v_cache"]))
    torch.cuda.synchronize()
    assert int(status.item()) == jsv.JSV_ERR_DEVICE_INPUT
