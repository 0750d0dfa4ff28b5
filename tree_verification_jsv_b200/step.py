"""One verify step on the device: buffers plus the four C-ABI calls.

``VerifyStep`` owns the device buffers for a fixed geometry (torch is used
for allocation and streams only) and issues, on one stream and with no host
synchronisation, the calls of ``include/jsv.h`` in order: tree attention,
LM head + argmax, and the accept walk with the KV compaction (one launch,
``jsv_accept_compact``; the separate ``jsv_accept_path`` and
``jsv_kv_compact`` are kept as methods too).

``run_host`` is the end-to-end form: it copies the step's per-step inputs
from pinned host memory, runs the step, and copies the accepted paths back.
The per-step inputs (tree arrays, tokens, q, hidden) live in one device
arena and the outputs (paths, lengths) in another, each mirrored by one
pinned host buffer, so each direction is a single copy.

``capture`` records the step's calls once into a CUDA graph (the engine the
JetSpec README describes replays CUDA graphs for wall-clock latency); every
kernel is launched with programmatic dependent launch, so the graph keeps
those overlapping edges.  ``replay`` launches the whole step in one call;
``capture_host`` / ``replay_host`` do the same for the end-to-end form,
copies included.
"""
from __future__ import annotations

import numpy as np
import torch

from . import jsv


def _i32(x, device):
    return torch.as_tensor(np.ascontiguousarray(x, dtype=np.int32)).to(device)


def _bf16(bits, device):
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(device)


class _Arena:
    """Named arrays packed at 256-byte offsets in one device buffer, with a
    pinned host mirror; ``dev[name]`` / ``host[name]`` are typed views."""

    def __init__(self, fields, device):
        # fields: name -> (shape, torch dtype)
        self.layout, off = {}, 0
        for name, (shape, dtype) in fields.items():
            n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
            self.layout[name] = (off, n, shape, dtype)
            off += (n + 255) // 256 * 256
        self.nbytes = max(off, 256)
        self.dev_buf = torch.zeros(self.nbytes, dtype=torch.uint8, device=device)
        self.host_buf = torch.zeros(self.nbytes, dtype=torch.uint8).pin_memory()
        self.dev = {k: self._view(self.dev_buf, k) for k in self.layout}
        self.host = {k: self._view(self.host_buf, k) for k in self.layout}

    def _view(self, buf, name):
        off, n, shape, dtype = self.layout[name]
        return buf[off:off + n].view(dtype).view(shape)


class VerifyStep:
    """Device state for one verify step of a workload (see ``synth.Workload``)."""

    def __init__(self, wl, tokens, device="cuda", max_path=None):
        dev = torch.device(device)
        self.device = dev
        self.B, self.Hq, self.Hkv, self.D = wl.B, wl.Hq, wl.Hkv, wl.D
        self.T, self.d, self.V = wl.T, wl.d, wl.V
        self.scale = wl.scale
        self.max_path = int(max_path or wl.max_nodes)
        # per-step inputs in one arena (filled once here from the workload)
        inputs = {"page_table": np.ascontiguousarray(wl.page_table, dtype=np.int32),
                  "prefix_len": np.ascontiguousarray(wl.prefix_len, dtype=np.int32),
                  "node_offsets": np.ascontiguousarray(wl.node_offsets, dtype=np.int32),
                  "parent": np.ascontiguousarray(wl.parent, dtype=np.int32),
                  "tokens": np.ascontiguousarray(tokens, dtype=np.int32),
                  "q": np.ascontiguousarray(wl.q, dtype=np.uint16),
                  "hidden": np.ascontiguousarray(wl.hidden, dtype=np.uint16)}
        self._in = _Arena({k: (v.shape, torch.int32 if v.dtype == np.int32 else torch.bfloat16)
                           for k, v in inputs.items()}, dev)
        for k, v in inputs.items():
            hv = self._in.host[k]
            if v.dtype == np.int32:
                hv.copy_(torch.from_numpy(v))
            else:
                hv.view(torch.int16).copy_(torch.from_numpy(v.view(np.int16)))
        self._in.dev_buf.copy_(self._in.host_buf)
        for k, t in self._in.dev.items():
            setattr(self, k, t)
        self.k_cache = _bf16(wl.k_cache, dev)
        self.v_cache = _bf16(wl.v_cache, dev)
        self.w = _bf16(wl.w, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.out = torch.empty((self.T, self.Hq, self.D), dtype=torch.bfloat16, device=dev)
        self.argmax = torch.empty(self.T, dtype=torch.int32, device=dev)
        self.max_logit = torch.empty(self.T, dtype=torch.float32, device=dev)
        # per-step outputs in one arena
        self._out = _Arena({"path": ((self.B, self.max_path), torch.int32), "accept_len": ((self.B,), torch.int32),
                            "bonus": ((self.B,), torch.int32), "new_len": ((self.B,), torch.int32)}, dev)
        for k, t in self._out.dev.items():
            setattr(self, k, t)
        self.batch = jsv.make_batch(
            B=self.B, Hq=self.Hq, Hkv=self.Hkv, D=self.D,
            max_pages_per_req=wl.page_table.shape[1], num_pages=wl.num_pages,
            total_nodes=self.T, max_nodes=wl.max_nodes, max_prefix=wl.max_prefix,
            page_table=self.page_table, prefix_len=self.prefix_len,
            node_offsets=self.node_offsets, parent=self.parent, dev_status=self.status)
        aws = jsv.jsv_tree_attention_workspace_size(self.batch)
        lws = jsv.jsv_lmhead_argmax_workspace_size(self.T, self.d, self.V)
        self.attn_ws = torch.zeros(max(aws, 256), dtype=torch.uint8, device=dev)   # any contents: every call writes what it reads
        self.lm_ws = torch.zeros(max(lws, 8), dtype=torch.uint8, device=dev)   # zeroed once; each call leaves it zeroed
        self._graph = None
        self._host_graph = None

    # -- the four calls -----------------------------------------------------
    def attention(self, stream=None):
        jsv.jsv_tree_attention(self.batch, self.q, self.k_cache, self.v_cache, self.scale,
                               self.out, self.attn_ws, stream=stream)

    def lmhead(self, stream=None):
        jsv.jsv_lmhead_argmax(self.hidden, self.w, self.T, self.d, self.V, self.argmax,
                              self.max_logit, self.lm_ws, dev_status=self.status, stream=stream)

    def accept(self, stream=None):
        jsv.jsv_accept_path(self.batch, self.tokens, self.argmax, self.max_path, self.path,
                            self.accept_len, self.bonus, stream=stream)

    def compact(self, stream=None):
        jsv.jsv_kv_compact(self.batch, self.k_cache, self.v_cache, self.path, self.max_path,
                           self.accept_len, self.new_len, stream=stream)

    def accept_compact(self, stream=None):
        """The walk and the compaction in one launch (same results as
        ``accept`` followed by ``compact``)."""
        jsv.jsv_accept_compact(self.batch, self.tokens, self.argmax, self.max_path, self.path,
                               self.accept_len, self.bonus, self.k_cache, self.v_cache, self.new_len,
                               stream=stream)

    def run(self, stream=None):
        """One verify step on one stream, no host sync: tree attention, LM head
        + argmax, then the accept walk fused with the KV compaction."""
        self.attention(stream)
        self.lmhead(stream)
        self.accept_compact(stream)

    # -- CUDA graph -----------------------------------------------------------
    def capture(self):
        """Record one verify step into a CUDA graph on a side stream.

        One eager step runs first so that every one-time host set-up (kernel
        attributes, tensor-map entry point) happens outside the capture; it
        executes the step, so callers that need pristine caches restore them
        before replaying."""
        self.run()
        torch.cuda.synchronize(self.device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.run()
        torch.cuda.synchronize(self.device)
        self._graph = graph
        return graph

    def replay(self):
        """One verify step through the captured graph (same buffers)."""
        self._graph.replay()

    # -- end-to-end form ----------------------------------------------------
    def host_inputs(self):
        """Pinned host views of the per-step inputs (tree arrays, tokens, q,
        hidden); ``run_host`` copies all of them in one transfer."""
        return self._in.host

    def h2d_bytes(self) -> int:
        return self._in.nbytes

    def d2h_bytes(self) -> int:
        return self._out.nbytes

    def run_host(self, stream=None):
        """Copy the input arena host->device, run the step, copy the output
        arena back (one copy each way); returns pinned host views of path,
        accept_len, bonus and new_len."""
        self._in.dev_buf.copy_(self._in.host_buf, non_blocking=True)
        self.run(stream)
        self._out.host_buf.copy_(self._out.dev_buf, non_blocking=True)
        return self._out.host

    def capture_host(self):
        """Record the end-to-end step (the input arena's copy up from pinned
        host memory, the step's calls, the output arena's copy back) into one
        CUDA graph, so that ``replay_host`` issues all of it with one launch.
        The graph's copies read and write the pinned buffers when it runs:
        the caller fills ``host_inputs()`` before each replay and reads the
        returned views after synchronising.  One eager ``run_host`` runs
        first (one-time host set-up outside the capture)."""
        self.run_host()
        torch.cuda.synchronize(self.device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.run_host()
        torch.cuda.synchronize(self.device)
        self._host_graph = graph
        return graph

    def replay_host(self):
        """One end-to-end step through the graph of ``capture_host``; returns
        the pinned host views of path, accept_len, bonus and new_len (filled
        once the current stream has been synchronised)."""
        self._host_graph.replay()
        return self._out.host
