"""One verify step on the device: buffers plus the four C-ABI calls.

``VerifyStep`` owns the device buffers for a fixed geometry (torch is used
for allocation and streams only) and issues, on one stream and with no host
synchronisation, the four calls of ``include/jsv.h`` in order:
tree attention, LM head + argmax, accept walk, KV compaction.

``run_host`` is the end-to-end form: it copies the step's per-step inputs
from pinned host memory, runs the step, and copies the accepted paths back.

``capture`` records the four calls once into a CUDA graph (the engine the
JetSpec README describes replays CUDA graphs for wall-clock latency); every
kernel is launched with programmatic dependent launch, so the graph keeps
those overlapping edges.  ``replay`` launches the whole step in one call.
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


class VerifyStep:
    """Device state for one verify step of a workload (see ``synth.Workload``)."""

    def __init__(self, wl, tokens, device="cuda", max_path=None):
        dev = torch.device(device)
        self.device = dev
        self.B, self.Hq, self.Hkv, self.D = wl.B, wl.Hq, wl.Hkv, wl.D
        self.T, self.d, self.V = wl.T, wl.d, wl.V
        self.scale = wl.scale
        self.max_path = int(max_path or wl.max_nodes)
        self.page_table = _i32(wl.page_table, dev)
        self.prefix_len = _i32(wl.prefix_len, dev)
        self.node_offsets = _i32(wl.node_offsets, dev)
        self.parent = _i32(wl.parent, dev)
        self.tokens = _i32(tokens, dev)
        self.q = _bf16(wl.q, dev)
        self.k_cache = _bf16(wl.k_cache, dev)
        self.v_cache = _bf16(wl.v_cache, dev)
        self.hidden = _bf16(wl.hidden, dev)
        self.w = _bf16(wl.w, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.out = torch.empty((self.T, self.Hq, self.D), dtype=torch.bfloat16, device=dev)
        self.argmax = torch.empty(self.T, dtype=torch.int32, device=dev)
        self.max_logit = torch.empty(self.T, dtype=torch.float32, device=dev)
        self.path = torch.empty((self.B, self.max_path), dtype=torch.int32, device=dev)
        self.accept_len = torch.empty(self.B, dtype=torch.int32, device=dev)
        self.bonus = torch.empty(self.B, dtype=torch.int32, device=dev)
        self.new_len = torch.empty(self.B, dtype=torch.int32, device=dev)
        self.batch = jsv.make_batch(
            B=self.B, Hq=self.Hq, Hkv=self.Hkv, D=self.D,
            max_pages_per_req=wl.page_table.shape[1], num_pages=wl.num_pages,
            total_nodes=self.T, max_nodes=wl.max_nodes, max_prefix=wl.max_prefix,
            page_table=self.page_table, prefix_len=self.prefix_len,
            node_offsets=self.node_offsets, parent=self.parent, dev_status=self.status)
        aws = jsv.jsv_tree_attention_workspace_size(self.batch)
        lws = jsv.jsv_lmhead_argmax_workspace_size(self.T, self.d, self.V)
        self.attn_ws = torch.empty(max(aws, 256), dtype=torch.uint8, device=dev)
        self.lm_ws = torch.empty(max(lws, 8), dtype=torch.uint8, device=dev)
        self._pinned = None
        self._graph = None

    # -- the four calls -----------------------------------------------------
    def attention(self, stream=None):
        jsv.jsv_tree_attention(self.batch, self.q, self.k_cache, self.v_cache, self.scale,
                               self.out, self.attn_ws, stream=stream)

    def lmhead(self, stream=None):
        jsv.jsv_lmhead_argmax(self.hidden, self.w, self.T, self.d, self.V, self.argmax,
                              self.max_logit, self.lm_ws, stream=stream)

    def accept(self, stream=None):
        jsv.jsv_accept_path(self.batch, self.tokens, self.argmax, self.max_path, self.path,
                            self.accept_len, self.bonus, stream=stream)

    def compact(self, stream=None):
        jsv.jsv_kv_compact(self.batch, self.k_cache, self.v_cache, self.path, self.max_path,
                           self.accept_len, self.new_len, stream=stream)

    def run(self, stream=None):
        """One verify step: four launches sequences on one stream, no host sync."""
        self.attention(stream)
        self.lmhead(stream)
        self.accept(stream)
        self.compact(stream)

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
        """Pinned host copies of the per-step inputs (tree, tokens, q, hidden)."""
        if self._pinned is None:
            self._pinned = {k: getattr(self, k).cpu().pin_memory()
                            for k in ("page_table", "prefix_len", "node_offsets", "parent",
                                      "tokens", "q", "hidden")}
            self._pinned_out = {k: torch.empty_like(getattr(self, k), device="cpu").pin_memory()
                                for k in ("path", "accept_len", "bonus", "new_len")}
        return self._pinned

    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.host_inputs().values())

    def d2h_bytes(self) -> int:
        self.host_inputs()
        return sum(t.numel() * t.element_size() for t in self._pinned_out.values())

    def run_host(self, stream=None):
        """Copy inputs host->device, run the step, copy the results back."""
        src = self.host_inputs()
        for k, t in src.items():
            getattr(self, k).copy_(t, non_blocking=True)
        self.run(stream)
        for k, t in self._pinned_out.items():
            t.copy_(getattr(self, k), non_blocking=True)
        return self._pinned_out
