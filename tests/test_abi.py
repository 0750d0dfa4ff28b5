"""The C-ABI library builds, loads, exports every declared symbol, and
rejects bad host-side arguments before touching a GPU (no compute calls)."""
import ctypes
import re
from pathlib import Path

import pytest

from tree_verification_jsv_b200 import build as jbuild
from tree_verification_jsv_b200 import jsv

ROOT = Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def lib():
    jbuild.build()
    return jsv.load()


def declared_symbols():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        names |= set(re.findall(r"JSV_API\s+[\w\s\*]+?\b(jsv_\w+)\s*\(", h.read_text()))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert {"jsv_tree_attention", "jsv_lmhead_argmax", "jsv_accept_path", "jsv_kv_compact"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert set(jsv.EXPORTS) <= names


def test_version_and_status_strings(lib):
    assert jsv.jsv_version() >= 100
    assert jsv.status_string(0) == "ok"
    assert "unsupported" in jsv.status_string(2)


def _batch(**kw):
    base = dict(B=1, Hq=4, Hkv=2, D=128, max_pages_per_req=4, num_pages=4, total_nodes=8,
                max_nodes=8, max_prefix=32, page_table=16, prefix_len=16, node_offsets=16,
                parent=16)
    base.update(kw)
    return jsv.make_batch(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), jsv.JSV_ERR_UNSUPPORTED),
    (dict(page_size=32), jsv.JSV_ERR_UNSUPPORTED),
    (dict(max_nodes=513), jsv.JSV_ERR_UNSUPPORTED),
    (dict(Hq=6, Hkv=4), jsv.JSV_ERR_INVALID_ARG),
    (dict(B=0), jsv.JSV_ERR_INVALID_ARG),
    (dict(total_nodes=0), jsv.JSV_ERR_INVALID_ARG),
    (dict(parent=None), jsv.JSV_ERR_INVALID_ARG),
])
def test_host_validation_rejects_batches(lib, kw, code):
    b = _batch(**kw)
    st = lib.jsv_tree_attention(ctypes.byref(b), 16, 16, 16, 0.1, 16, 256, 1 << 30, None)
    assert st == code
    st = lib.jsv_accept_path(ctypes.byref(b), 16, 16, 8, 16, 16, 16, None)
    assert st == code
    st = lib.jsv_kv_compact(ctypes.byref(b), 16, 16, 16, 8, 16, 16, None)
    assert st == code
    st = lib.jsv_accept_compact(ctypes.byref(b), 16, 16, 8, 16, 16, 16, 16, 16, 16, None)
    assert st == code


def test_host_validation_other_arguments(lib):
    b = _batch()
    # NULL output, misaligned q, bad scale, too-small workspace
    assert lib.jsv_tree_attention(ctypes.byref(b), 16, 16, 16, 0.1, None, 256, 1 << 30, None) == 1
    assert lib.jsv_tree_attention(ctypes.byref(b), 18, 16, 16, 0.1, 16, 256, 1 << 30, None) == 1
    assert lib.jsv_tree_attention(ctypes.byref(b), 16, 16, 16, -1.0, 16, 256, 1 << 30, None) == 1
    assert lib.jsv_tree_attention(ctypes.byref(b), 16, 16, 16, 0.1, 16, 256, 1, None) == 1
    assert lib.jsv_tree_attention_workspace_size(ctypes.byref(b)) > 0
    assert lib.jsv_accept_path(ctypes.byref(b), 16, 16, 0, 16, 16, 16, None) == 1
    assert lib.jsv_accept_compact(ctypes.byref(b), 16, 16, 0, 16, 16, 16, 16, 16, 16, None) == 1
    assert lib.jsv_accept_compact(ctypes.byref(b), 16, 16, 8, 16, 16, 16, 18, 16, 16, None) == 1
    # LM head: d not a multiple of 64, missing workspace, NULL output
    assert lib.jsv_lmhead_argmax(16, 16, 4, 100, 50, 16, None, 16, 1 << 20, None, None) == 2
    assert lib.jsv_lmhead_argmax(16, 16, 4, 128, 50, 16, None, None, 0, None, None) == 1
    assert lib.jsv_lmhead_argmax(16, 16, 4, 128, 50, None, None, 16, 1 << 20, None, None) == 1
    assert lib.jsv_lmhead_argmax_workspace_size(4, 128, 50) >= 32
    # bounded-wait self-test: NULL status word, limits out of range
    assert lib.jsv_selftest_wait_timeout(None, 10, None) == 1
    assert lib.jsv_selftest_wait_timeout(16, 0, None) == 1
    assert lib.jsv_selftest_wait_timeout(16, 3_000_000, None) == 1
    # LM-head timeout self-test: status word required, limit in range, the
    # workspace or the no-alloc limit checked like the entry point it mimics
    big = jsv.NOALLOC_MAX_NODES + 1
    assert lib.jsv_selftest_lmhead_timeout(16, 16, 4, 128, 50, 16, None, 16, 1 << 20, None, 10, None) == 1
    assert lib.jsv_selftest_lmhead_timeout(16, 16, 4, 128, 50, 16, None, 16, 1 << 20, 16, 0, None) == 1
    assert lib.jsv_selftest_lmhead_timeout(16, 16, 4, 128, 50, 16, None, 16, 1, 16, 10, None) == 1
    assert lib.jsv_selftest_lmhead_timeout(16, 16, big, 128, 50, 16, None, None, 0, 16, 10, None) == 2
    assert lib.jsv_selftest_lmhead_timeout(16, 16, 4, 100, 50, 16, None, None, 0, 16, 10, None) == 2
    # the no-alloc entry point: the node limit and the LM head's own checks
    assert lib.jsv_lmhead_argmax_noalloc(16, 16, big, 128, 50, 16, None, None, None) == 2
    assert lib.jsv_lmhead_argmax_noalloc(16, 16, 4, 100, 50, 16, None, None, None) == 2
    assert lib.jsv_lmhead_argmax_noalloc(16, 16, 4, 128, 50, None, None, None, None) == 1


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(jsv, "_SO", tmp_path / "missing.so")
    monkeypatch.setattr(jsv, "_lib", None)
    with pytest.raises(RuntimeError):
        jsv.load()


def test_checked_build_exports_the_same_symbols_and_says_so(lib):
    """libjsv_checked.so (-DJSV_CHECK_BOUNDS) exports every declared symbol
    and reports its build flag; the ordinary library reports none."""
    so = jbuild.build(checked=True)
    chk = ctypes.CDLL(str(so))
    for n in declared_symbols():
        assert hasattr(chk, n), n
    chk.jsv_build_flags.restype = ctypes.c_int32
    assert chk.jsv_build_flags() & 1 == 1
    assert jsv.jsv_build_flags() & 1 == 0
    chk.jsv_status_string.restype = ctypes.c_char_p
    assert b"bounds" in chk.jsv_status_string(jsv.JSV_ERR_BOUNDS)
