"""ctypes binding of libjsv.so (argument marshalling only).

Every function has the name of the C entry point it calls (``include/jsv.h``)
and takes torch tensors (or raw integer device addresses).  There is no
fallback: if ``libjsv.so`` is missing or fails to load, every call raises.
Build it with ``python -m tree_verification_jsv_b200.build``.

With ``JSV_LIBRARY=checked`` in the environment the binding loads the
checked build, ``libjsv_checked.so`` (every computed global index checked,
misses reported as JSV_ERR_BOUNDS), from the same directory instead.
"""
from __future__ import annotations

import ctypes
import os
from pathlib import Path

_DIR = Path(__file__).resolve().parent
_SO = _DIR / ("libjsv_checked.so" if os.environ.get("JSV_LIBRARY") == "checked" else "libjsv.so")
_lib = None

JSV_OK = 0
JSV_ERR_INVALID_ARG = 1
JSV_ERR_UNSUPPORTED = 2
JSV_ERR_CUDA = 3
JSV_ERR_TIMEOUT = 4
JSV_ERR_DEVICE_INPUT = 5
JSV_ERR_BOUNDS = 6

EXPORTS = ("jsv_tree_attention_workspace_size", "jsv_tree_attention",
           "jsv_lmhead_argmax_workspace_size", "jsv_lmhead_argmax", "jsv_accept_path",
           "jsv_kv_compact", "jsv_status_string", "jsv_version", "jsv_kernel_launches",
           "jsv_lmhead_argmax_noalloc", "jsv_last_error_string", "jsv_selftest_wait_timeout",
           "jsv_selftest_lmhead_timeout",
           "jsv_accum_logp_tree", "jsv_tree_qkv_rope", "jsv_accept_compact", "jsv_build_flags")

# Largest node count jsv_lmhead_argmax_noalloc accepts (JSV_NOALLOC_MAX_NODES).
NOALLOC_MAX_NODES = 8192


class JsvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = f"{fn}: {status_string(status)} (status {status})"
        if status == JSV_ERR_CUDA:
            msg += f": {load().jsv_last_error_string().decode()}"
        super().__init__(msg)
        self.status = status


class jsv_batch(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("D", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_pages_per_req", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("total_nodes", ctypes.c_int32), ("max_nodes", ctypes.c_int32),
                ("max_prefix", ctypes.c_int32),
                ("page_table", ctypes.c_void_p), ("prefix_len", ctypes.c_void_p),
                ("node_offsets", ctypes.c_void_p), ("parent", ctypes.c_void_p),
                ("dev_status", ctypes.c_void_p)]


def library_path() -> Path:
    return _SO


def load() -> ctypes.CDLL:
    """Load libjsv.so once; raises if it is missing (no CPU fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not _SO.exists():
        raise RuntimeError(f"{_SO.name} not built at {_SO}; run python -m tree_verification_jsv_b200.build")
    lib = ctypes.CDLL(str(_SO))
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    bp = ctypes.POINTER(jsv_batch)
    lib.jsv_tree_attention_workspace_size.argtypes = [bp]
    lib.jsv_tree_attention_workspace_size.restype = sz
    lib.jsv_tree_attention.argtypes = [bp, vp, vp, vp, ctypes.c_float, vp, vp, sz, vp]
    lib.jsv_tree_attention.restype = ctypes.c_int
    lib.jsv_lmhead_argmax_workspace_size.argtypes = [i32, i32, i32]
    lib.jsv_lmhead_argmax_workspace_size.restype = sz
    lib.jsv_lmhead_argmax.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, sz, vp, vp]
    lib.jsv_lmhead_argmax.restype = ctypes.c_int
    lib.jsv_accept_path.argtypes = [bp, vp, vp, i32, vp, vp, vp, vp]
    lib.jsv_accept_path.restype = ctypes.c_int
    lib.jsv_kv_compact.argtypes = [bp, vp, vp, vp, i32, vp, vp, vp]
    lib.jsv_kv_compact.restype = ctypes.c_int
    lib.jsv_accept_compact.argtypes = [bp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.jsv_accept_compact.restype = ctypes.c_int
    lib.jsv_status_string.argtypes = [ctypes.c_int]
    lib.jsv_status_string.restype = ctypes.c_char_p
    lib.jsv_version.argtypes = []
    lib.jsv_version.restype = i32
    lib.jsv_build_flags.argtypes = []
    lib.jsv_build_flags.restype = i32
    lib.jsv_lmhead_argmax_noalloc.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, vp]
    lib.jsv_lmhead_argmax_noalloc.restype = ctypes.c_int
    lib.jsv_tree_qkv_rope.argtypes = [bp, vp, vp, i32, vp, vp, i32, vp, vp, vp, vp]
    lib.jsv_tree_qkv_rope.restype = ctypes.c_int
    lib.jsv_accum_logp_tree.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.jsv_accum_logp_tree.restype = ctypes.c_int
    lib.jsv_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint32, vp]
    lib.jsv_selftest_wait_timeout.restype = ctypes.c_int
    lib.jsv_selftest_lmhead_timeout.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp, sz, vp, ctypes.c_uint32, vp]
    lib.jsv_selftest_lmhead_timeout.restype = ctypes.c_int
    lib.jsv_last_error_string.argtypes = []
    lib.jsv_last_error_string.restype = ctypes.c_char_p
    lib.jsv_kernel_launches.argtypes = []
    lib.jsv_kernel_launches.restype = ctypes.c_uint64
    _lib = lib
    return lib


def _addr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, st: int) -> None:
    if st != JSV_OK:
        raise JsvError(fn, st)


def status_string(status: int) -> str:
    return load().jsv_status_string(int(status)).decode()


def jsv_version() -> int:
    return int(load().jsv_version())


def jsv_build_flags() -> int:
    """Bit 0: the loaded library is the checked build (JSV_CHECK_BOUNDS)."""
    return int(load().jsv_build_flags())


def jsv_kernel_launches() -> int:
    return int(load().jsv_kernel_launches())


def make_batch(*, B, Hq, Hkv, D, max_pages_per_req, num_pages, total_nodes, max_nodes,
               max_prefix, page_table, prefix_len, node_offsets, parent, dev_status=None,
               page_size=16) -> jsv_batch:
    return jsv_batch(int(B), int(Hq), int(Hkv), int(D), int(page_size), int(max_pages_per_req),
                     int(num_pages), int(total_nodes), int(max_nodes), int(max_prefix),
                     _addr(page_table), _addr(prefix_len), _addr(node_offsets), _addr(parent),
                     _addr(dev_status))


def jsv_tree_attention_workspace_size(batch: jsv_batch) -> int:
    return int(load().jsv_tree_attention_workspace_size(ctypes.byref(batch)))


def jsv_tree_attention(batch, q, k_cache, v_cache, scale, out, workspace, workspace_bytes=None,
                       stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().jsv_tree_attention(ctypes.byref(batch), _addr(q), _addr(k_cache), _addr(v_cache),
                                   float(scale), _addr(out), _addr(workspace), int(workspace_bytes),
                                   _stream(stream))
    _check("jsv_tree_attention", st)


def jsv_lmhead_argmax_workspace_size(T, d, V) -> int:
    return int(load().jsv_lmhead_argmax_workspace_size(int(T), int(d), int(V)))


def _nbytes(buf, nbytes):
    if nbytes is not None:
        return int(nbytes)
    return 0 if buf is None or isinstance(buf, int) else buf.numel() * buf.element_size()


def jsv_lmhead_argmax(hidden, w, T, d, V, argmax, max_logit, workspace, workspace_bytes=None,
                      dev_status=None, stream=None) -> None:
    st = load().jsv_lmhead_argmax(_addr(hidden), _addr(w), int(T), int(d), int(V), _addr(argmax),
                                  _addr(max_logit), _addr(workspace), _nbytes(workspace, workspace_bytes),
                                  _addr(dev_status), _stream(stream))
    _check("jsv_lmhead_argmax", st)


def jsv_lmhead_argmax_noalloc(hidden, w, T, d, V, argmax, max_logit, dev_status=None, stream=None) -> None:
    """LM-head argmax with the library's fixed scratch (no workspace, no
    allocation); see include/jsv.h for its limits and sharing rules."""
    st = load().jsv_lmhead_argmax_noalloc(_addr(hidden), _addr(w), int(T), int(d), int(V),
                                          _addr(argmax), _addr(max_logit), _addr(dev_status), _stream(stream))
    _check("jsv_lmhead_argmax_noalloc", st)


def jsv_selftest_lmhead_timeout(hidden, w, T, d, V, argmax, max_logit, workspace, dev_status, limit_us,
                                workspace_bytes=None, stream=None) -> None:
    """The LM head with one injected wait that gives up (see include/jsv.h);
    ``workspace=None`` runs it on the no-alloc entry point's scratch array."""
    st = load().jsv_selftest_lmhead_timeout(_addr(hidden), _addr(w), int(T), int(d), int(V), _addr(argmax),
                                            _addr(max_logit), _addr(workspace), _nbytes(workspace, workspace_bytes),
                                            _addr(dev_status), int(limit_us), _stream(stream))
    _check("jsv_selftest_lmhead_timeout", st)


def jsv_tree_qkv_rope(batch, x, w_qkv, d, rope_cos, rope_sin, max_pos, q, k_cache, v_cache,
                      stream=None) -> None:
    st = load().jsv_tree_qkv_rope(ctypes.byref(batch), _addr(x), _addr(w_qkv), int(d), _addr(rope_cos),
                                  _addr(rope_sin), int(max_pos), _addr(q), _addr(k_cache), _addr(v_cache),
                                  _stream(stream))
    _check("jsv_tree_qkv_rope", st)


def jsv_accum_logp_tree(logp, topk_tokens, root_token, B, depth, width, budget, parent, tokens,
                        node_depth, score, num_nodes, dev_status=None, stream=None) -> None:
    st = load().jsv_accum_logp_tree(_addr(logp), _addr(topk_tokens), _addr(root_token), int(B), int(depth),
                                    int(width), int(budget), _addr(parent), _addr(tokens), _addr(node_depth),
                                    _addr(score), _addr(num_nodes), _addr(dev_status), _stream(stream))
    _check("jsv_accum_logp_tree", st)


def jsv_selftest_wait_timeout(dev_status, limit_us, stream=None) -> None:
    """Launch the bounded-wait self-test (see include/jsv.h)."""
    st = load().jsv_selftest_wait_timeout(_addr(dev_status), int(limit_us), _stream(stream))
    _check("jsv_selftest_wait_timeout", st)


def jsv_accept_path(batch, tokens, argmax, max_path, path, accept_len, bonus, stream=None) -> None:
    st = load().jsv_accept_path(ctypes.byref(batch), _addr(tokens), _addr(argmax), int(max_path),
                                _addr(path), _addr(accept_len), _addr(bonus), _stream(stream))
    _check("jsv_accept_path", st)


def jsv_kv_compact(batch, k_cache, v_cache, path, max_path, accept_len, new_len,
                   stream=None) -> None:
    st = load().jsv_kv_compact(ctypes.byref(batch), _addr(k_cache), _addr(v_cache), _addr(path),
                               int(max_path), _addr(accept_len), _addr(new_len), _stream(stream))
    _check("jsv_kv_compact", st)


def jsv_accept_compact(batch, tokens, argmax, max_path, path, accept_len, bonus, k_cache, v_cache, new_len,
                       stream=None) -> None:
    st = load().jsv_accept_compact(ctypes.byref(batch), _addr(tokens), _addr(argmax), int(max_path),
                                   _addr(path), _addr(accept_len), _addr(bonus), _addr(k_cache),
                                   _addr(v_cache), _addr(new_len), _stream(stream))
    _check("jsv_accept_compact", st)
