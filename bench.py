#!/usr/bin/env python
"""Benchmark of the one-forward tree verification step; prints ONE JSON line.

A step is one pass of the whole hot path over one batch of synthetic input:
tree attention, LM head + argmax, accept walk and KV compaction, i.e. the
calls of ``include/jsv.h`` on one stream (the walk and the compaction as the
one fused ``jsv_accept_compact`` launch).  Inputs are resident in HBM
when the timed region starts; L2 is flushed before every timed step,
outside its events: a write of four times the device's L2 (its size read
from the device), then a read of the same buffer, so the flush's own dirty
lines go back to HBM before the step rather than inside it.  Steps are
timed one by one with CUDA events on the launching stream; the headline is
the median step (p10, p90 and the mean beside it).  A second timed pass of
the same steps puts an event between the calls for the per-call durations
(the roofline).

The headline workload (``--workload``, default the Qwen3-8B-shaped 64-node
tree) is timed over exactly ``--steps`` steps.  On one GPU the line also
carries a ``workloads`` object with every other named workload, each timed
over at least 50 steps the same way and checked against its stored oracle
values (argmax, accept lengths, bonus tokens).

``e2e`` is the same metric through the public step API with host buffers:
per step, one copy of the step's inputs up from pinned host memory, the
step, one copy of the outputs back, and a host synchronisation, timed by
the host clock.  It is taken through ``VerifyStep.replay_host`` (the copies
and calls replayed from one CUDA graph, as a serving engine runs the step);
``e2e.eager`` gives ``VerifyStep.run_host`` (the calls issued from Python
every step), which is also the ``e2e`` figure under ``--no-graph``.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

Multi-GPU: the path does not shard inside one step (replicas only), so
under torchrun every rank runs its own replica of the workload; the value is
all ranks' nodes divided by the slowest rank's time (weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time
from datetime import timedelta
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "verified tree nodes/sec & verify-step latency; achieved HBM GB/s vs roofline"

DESCRIPTION = {
    "tiny": "tiny: 1 request, 2 q heads / 1 kv head, head_dim 64, hidden 256, vocab 1024, prefix 128, 16-node tree",
    "8b_64": "Qwen3-8B-shaped single request: 32q/8kv heads, head_dim 128, hidden 4096, vocab 151936, prefix 2048, 64-node tree (depth 8, top-4)",
    "8b_256": "Qwen3-8B-shaped long context: 32q/8kv, head_dim 128, hidden 4096, vocab 151936, prefix 16384, 256-node tree (depth 16, top-8)",
    "ragged16": "ragged batch of 16, Qwen3-8B shapes: prefixes U[512,8192], 32-128-node trees of depth 4-12",
    "30b_512x4": "Qwen3-30B-A3B-shaped: 32q/4kv, head_dim 128, hidden 2048, vocab 151936, batch 4, prefix 32768, 512-node trees (depth 16, top-8)",
}

# draft-tree shape of each workload for the tree-construction timing:
# (depth, width, budget) -- the pages' tree_depth / tree_width / budget
TREE_SHAPE = {"tiny": (5, 3, 16), "8b_64": (8, 4, 64), "8b_256": (16, 8, 256),
              "ragged16": (12, 4, 128), "30b_512x4": (16, 8, 512)}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["jsv", "reference"], default="jsv")
    ap.add_argument("--workload", default="8b_64", choices=list(DESCRIPTION))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--workloads", default="all",
                    help="comma-separated extra workloads timed on one GPU ('all', or 'none')")
    ap.add_argument("--profile", choices=["attention", "lmhead", "accept", "compact", "accept_compact", "tree", "qkv"],
                    help="run only this call K times after W warm-up (for ncu); prints its mean time")
    return ap.parse_args()


def tree_call(wl, st, dev):
    """A jsv_accum_logp_tree call on this workload's draft-tree shape (seeded top-k)."""
    import torch
    from tree_verification_jsv_b200 import jsv
    from tree_verification_jsv_b200 import synth as _synth
    Dt, kt, bt = TREE_SHAPE[wl.name]
    lp, tk, rt = _synth.draft_topk(wl.seed, wl.B, Dt, kt, wl.V)
    lp_d, tk_d, rt_d = (torch.as_tensor(x).to(dev) for x in (lp, tk, rt))
    tp = torch.empty((wl.B, bt), dtype=torch.int32, device=dev)
    ttok, tdep = torch.empty_like(tp), torch.empty_like(tp)
    tsc = torch.empty((wl.B, bt), dtype=torch.float32, device=dev)
    tnn = torch.empty(wl.B, dtype=torch.int32, device=dev)

    def call():
        jsv.jsv_accum_logp_tree(lp_d, tk_d, rt_d, wl.B, Dt, kt, bt, tp, ttok, tdep, tsc, tnn, st.status)
    return call


def qkv_rope_call(wl, st, dev):
    """A jsv_tree_qkv_rope call: seeded random-init fused Q/K/V weights, rotary base 1e6."""
    import torch
    from tree_verification_jsv_b200 import jsv
    from tree_verification_jsv_b200 import rope as _rope
    rows = (wl.Hq + 2 * wl.Hkv) * wl.D
    gq = torch.Generator(device=dev).manual_seed(wl.seed)
    w_qkv = (torch.randn(rows, wl.d, device=dev, generator=gq) / math.sqrt(wl.d)).to(torch.bfloat16)
    max_pos = wl.max_prefix + wl.max_nodes + 1
    cos_t, sin_t = (torch.as_tensor(t).to(dev) for t in _rope.rope_tables(1e6, wl.D, max_pos))

    def call():
        jsv.jsv_tree_qkv_rope(st.batch, st.hidden, w_qkv, wl.d, cos_t, sin_t, max_pos, st.q,
                              st.k_cache, st.v_cache)
    return call


def golden(name):
    return json.loads((ROOT / "tests" / "golden" / f"lmhead_{name}.json").read_text())


def load_workload(name):
    from tree_verification_jsv_b200 import synth
    g = golden(name)
    wl = synth.make_workload(name, redraws={int(k): v for k, v in g["redraws"].items()})
    return wl, np.asarray(g["tokens"], dtype=np.int32), g


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def workload_model(wl):
    """Algorithmic bytes / flops of each call and of the step."""
    kv_row = wl.Hkv * wl.D * 2                      # one slot of K (or V), bf16
    prefix = int(wl.prefix_len.sum())
    nodes = wl.T
    w_bytes = wl.V * wl.d * 2
    attn_bytes = 2 * kv_row * (prefix + nodes) + 2 * nodes * wl.Hq * wl.D * 2
    from tree_verification_jsv_b200 import synth
    vis = 0
    for b in range(wl.B):
        sl = wl.request_nodes(b)
        vis += int((wl.prefix_len[b] + synth.depths(wl.parent[sl]) + 1).sum())
    attn_flops = 4 * wl.Hq * wl.D * vis
    lm_bytes = w_bytes + nodes * wl.d * 2 + nodes * 8
    lm_flops = 2 * nodes * wl.d * wl.V
    return {
        "step_hbm_bytes": 2 * kv_row * prefix + w_bytes,
        "attention": {"bytes": attn_bytes, "flops": attn_flops},
        "lmhead": {"bytes": lm_bytes, "flops": lm_flops},
        "step_flops": attn_flops + lm_flops,
    }


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML about every
    millisecond by a background thread for the whole GPU arm.  ``region``
    records the host-time span of a timed region (launches plus the final
    synchronisation); ``summary`` reports the samples taken inside the named
    regions.  Without NVML the summary says so (source "unavailable")."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.period = period_s
        self.samples = []            # (host time, SM MHz, reasons bitmask)
        self.regions = {}            # name -> [(t0, t1), ...]
        self.max_mhz = None
        self.handle = None
        self._stop = threading.Event()
        self.thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nvml = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.handle = None

    def _poll(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                mhz = float(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM))
                r = int(n.nvmlDeviceGetCurrentClocksEventReasons(self.handle))
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.handle is not None and self.thread is None:
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
        return self

    def stop(self):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=2)
            self.thread = None

    class _Region:
        def __init__(self, owner, name):
            self.owner, self.name = owner, name

        def __enter__(self):
            self.t0 = time.perf_counter()
            return self

        def __exit__(self, *exc):
            self.owner.regions.setdefault(self.name, []).append((self.t0, time.perf_counter()))

    def region(self, name):
        return ClockSampler._Region(self, name)

    def summary(self, names=None):
        spans = [sp for k, v in self.regions.items() if names is None or k in names for sp in v]
        sel = [(m, r) for t, m, r in self.samples if any(a <= t <= b for a, b in spans)]
        reasons = sorted({name for _, r in sel for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median([m for m, _ in sel]) if sel else None,
                "sm_mhz_min": min(m for m, _ in sel) if sel else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(sel),
                "source": "nvml" if self.handle is not None else "unavailable"}


def step_stats(ms):
    """Median, p10, p90 and mean of per-step times (ms) in microseconds."""
    a = np.asarray(ms, dtype=np.float64) * 1e3
    return {"median": float(np.median(a)), "p10": float(np.percentile(a, 10)),
            "p90": float(np.percentile(a, 90)), "mean": float(a.mean()), "n": int(a.size)}


def accept_hist(accept_len):
    h = {}
    for a in accept_len:
        h[str(int(a))] = h.get(str(int(a)), 0) + 1
    return dict(sorted(h.items(), key=lambda kv: int(kv[0])))


def tpf_mean(hist):
    """Mean tokens per forward over the requests: accepted draft tokens plus
    the bonus token, a + 1 (the accept-length histogram counts a)."""
    n = sum(hist.values())
    return sum((int(a) + 1) * c for a, c in hist.items()) / n if n else None


def source_sha(*files):
    h = hashlib.sha256()
    for f in files:
        h.update((ROOT / f).read_bytes())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """DRAM bytes per launch (read + write) of the dominant kernel from the
    committed ncu summary -- only for the workload it was captured on and only
    while the kernel's source hash still matches (else None)."""
    p = ROOT / "profiles" / "ncu_traffic.json"
    if not p.exists():
        return None
    entries = json.loads(p.read_text()).get(kernel_key)
    if isinstance(entries, dict):
        entries = [entries]
    for d in entries or []:
        if d.get("workload") == workload and d.get("source_sha") == source_sha(*d["sources"]):
            return int(d["dram_bytes_per_launch"])
    return None


# ---------------------------------------------------------------------------
# Multi-rank aggregation (replicas only: no data-path collective)
# ---------------------------------------------------------------------------

def reduce_max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings over all ranks of the
    default process group (a no-op on one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_value(nodes_per_rank, world, ms_per_step_max):
    """Verified nodes per second of the whole job: every rank verifies its
    own replica's nodes in each step; the slowest rank sets the pace."""
    return world * nodes_per_rank / (ms_per_step_max * 1e-3)


# ---------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline leg)
# ---------------------------------------------------------------------------

def oracle_sample_step(wl, tokens, g, sample_nodes, threads=None):
    """The oracle's version of one step on a bounded sample: attention of
    every head of the first ``sample_nodes`` nodes of request 0, their LM-head
    argmax, and the walk + compaction of request 0.  Returns nodes done."""
    import oracle
    n0 = int(wl.node_offsets[1])
    ns = min(sample_nodes, n0)
    tt, hh = np.meshgrid(np.arange(ns), np.arange(wl.Hq), indexing="ij")
    rows = np.stack([tt.ravel(), hh.ravel()], axis=1)
    oracle.tree_attention_wl(wl, rows=rows, threads=threads)
    oracle.lmhead_top2(wl.hidden, wl.w, rows=np.arange(ns))
    arg = np.asarray(g["argmax"], dtype=np.int64)
    path, a, bonus = oracle.accept_path(wl.parent[:n0], tokens[:n0], arg[:n0])
    k = wl.k_cache.copy()
    v = wl.v_cache.copy()
    oracle.kv_compact(k, v, wl.page_table[:1], wl.prefix_len[:1], [path])
    return ns


def cpu_model():
    try:
        for line in Path("/proc/cpuinfo").read_text().splitlines():
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(wl, tokens, g, steps=1, sample_nodes=64):
    """The oracle on the host cores (its C attention on every core, numpy's
    BLAS for the LM head), plus single-thread figures for the tiny workload
    and for a 16-node sample of the Qwen3-8B-shaped 64-node one."""
    import oracle
    t0 = time.perf_counter()
    done = 0
    for _ in range(steps):
        done += oracle_sample_step(wl, tokens, g, sample_nodes)
    dt = time.perf_counter() - t0
    ns = min(sample_nodes, int(wl.node_offsets[1]))
    out = {"value": done / dt, "unit": "nodes/s", "cores": oracle.host_threads(),
           "kind": "oracle", "cpu_model": cpu_model(),
           "sample": f"{ns} nodes of request 0 (all {wl.Hq} heads' attention + LM-head argmax over "
                     f"{wl.V} tokens, fp64) + walk and KV compaction of request 0, x{steps}",
           "seconds": dt}
    single = {}
    try:
        from threadpoolctl import threadpool_limits
        for name, wl1, tok1, g1, n1 in (("tiny",) + load_workload("tiny") + (16,),
                                        (wl.name, wl, tokens, g, 16)):
            if name not in ("tiny", "8b_64"):
                continue
            with threadpool_limits(limits=1):
                t1 = time.perf_counter()
                d1 = oracle_sample_step(wl1, tok1, g1, n1, threads=1)
                single[name] = {"value": d1 / (time.perf_counter() - t1), "unit": "nodes/s",
                                "sample": f"{d1} nodes, one thread (oracle and BLAS)"}
    except ImportError:
        single = {"unavailable": "threadpoolctl missing"}
    out["single_thread"] = single
    return out


def run_reference(args, rank):
    """--impl reference: the oracle as it stands, on the host cores."""
    if rank != 0:
        return
    wl, tokens, g = load_workload(args.workload)
    sample = 16
    for _ in range(args.warmup):
        oracle_sample_step(wl, tokens, g, sample)
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += oracle_sample_step(wl, tokens, g, sample)
    dt = time.perf_counter() - t0
    import oracle
    value = done / dt
    ns = min(sample, int(wl.node_offsets[1]))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "nodes/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DESCRIPTION[args.workload], "name": args.workload,
                   "sample_nodes_per_step": ns, "l2": "n/a (host)"},
        "cpu_baseline": {"value": value, "unit": "nodes/s", "cores": oracle.host_threads(),
                         "kind": "oracle",
                         "sample": f"per step: {ns} nodes of request 0 (attention all heads + LM-head "
                                   f"argmax, fp64) + walk and compaction of request 0"},
        "e2e": {"value": value, "unit": "nodes/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

class GpuBench:
    """Timing helpers over one device: an L2 flush sized from the device,
    per-step CUDA events, the clock sampler."""

    def __init__(self, local_rank):
        import torch
        self.torch = torch
        self.dev = f"cuda:{local_rank}"
        props = torch.cuda.get_device_properties(local_rank)
        self.l2_bytes = int(props.L2_cache_size)
        self.flush_bytes = max(4 * self.l2_bytes, 64 << 20)
        self.flush = torch.empty(self.flush_bytes, dtype=torch.uint8, device=self.dev)
        self.stream = torch.cuda.current_stream()
        self.clocks = ClockSampler(local_rank).start()

    def flush_l2(self, i):
        # Write four times the L2, then read it back: the write evicts every
        # line of the step's data, and the read makes the flush's own dirty
        # lines go back to HBM here rather than inside the timed step.
        self.flush.fill_(i & 0xFF)
        self.flush.view(self.torch.int64).sum()

    def time_steps(self, fn, K, region):
        """Per-step device times (ms) of fn(), L2 flushed before each."""
        torch = self.torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        torch.cuda.synchronize()
        with self.clocks.region(region):
            for i in range(K):
                self.flush_l2(i)
                ev[i][0].record(self.stream)
                fn()
                ev[i][1].record(self.stream)
            torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def time_calls(self, st, K, region):
        """Per-call device times (ms) [K, 3]: attention, LM head, walk + compaction."""
        torch = self.torch
        evc = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
        torch.cuda.synchronize()
        with self.clocks.region(region):
            for i in range(K):
                self.flush_l2(i)
                e = evc[i]
                e[0].record(self.stream)
                st.attention()
                e[1].record(self.stream)
                st.lmhead()
                e[2].record(self.stream)
                st.accept_compact()
                e[3].record(self.stream)
            torch.cuda.synchronize()
        return np.array([[evc[i][j].elapsed_time(evc[i][j + 1]) for j in range(3)] for i in range(K)])


CALLS = ["attention", "lmhead", "accept_compact"]


def check_against_golden(st, g):
    """This launch configuration's outputs against the stored oracle values."""
    assert int(st.status.item()) == 0, "device-side error"
    assert st.argmax.cpu().numpy().tolist() == g["argmax"], "argmax differs from the oracle golden"
    assert st.accept_len.cpu().numpy().tolist() == g["accept_len"], "accept_len differs from the oracle"
    assert st.bonus.cpu().numpy().tolist() == g["bonus"], "bonus differs from the oracle"
    return {"argmax": "bit-exact vs oracle", "accept_len": "bit-exact vs oracle", "bonus": "bit-exact vs oracle"}


def fractions(model, step_us, hbm, tf_burst, tf_sus):
    t = step_us * 1e-6
    return {"step_hbm_gbs": model["step_hbm_bytes"] / t / 1e9,
            "step_hbm_frac": model["step_hbm_bytes"] / t / 1e9 / hbm,
            "step_tensor_frac": model["step_flops"] / t / 1e12 / tf_burst,
            "step_tensor_frac_sustained": model["step_flops"] / t / 1e12 / tf_sus}


def measure_workload(gb, name, K, warmup, pk):
    """One extra workload on this GPU: oracle check, then K whole steps and K
    steps with per-call events, L2 flushed before each."""
    import torch
    from tree_verification_jsv_b200.step import VerifyStep
    hbm, tf_burst, tf_sus, _ = pk
    wl, tokens, g = load_workload(name)
    st = VerifyStep(wl, tokens, device=gb.dev)
    st.run()
    torch.cuda.synchronize()
    check = check_against_golden(st, g)
    hist = accept_hist(st.accept_len.cpu().numpy())
    for _ in range(max(warmup, 3)):
        gb.flush_l2(1)
        st.run()
    torch.cuda.synchronize()
    steps = gb.time_steps(st.run, K, f"steps:{name}")
    per = gb.time_calls(st, K, f"calls:{name}")
    assert int(st.status.item()) == 0
    model = workload_model(wl)
    stat = step_stats(steps)
    out = {"workload": DESCRIPTION[name], "nodes": wl.T, "requests": wl.B,
           "prefix_tokens": int(wl.prefix_len.sum()), "steps": K, "step_us": stat,
           "nodes_per_s": wl.T / (stat["median"] * 1e-6),
           **fractions(model, stat["median"], hbm, tf_burst, tf_sus),
           "step_hbm_bytes": model["step_hbm_bytes"], "step_flops": model["step_flops"],
           "call_us": {n: float(np.median(per[:, j]) * 1e3) for j, n in enumerate(CALLS)},
           "clocks": gb.clocks.summary([f"steps:{name}", f"calls:{name}"]),
           "check": check, "accept_len_hist": hist, "tokens_per_forward_mean": tpf_mean(hist)}
    del st
    torch.cuda.empty_cache()
    return out


def run_gpu(args, rank, world, local_rank):
    import torch
    from tree_verification_jsv_b200 import jsv
    from tree_verification_jsv_b200.step import VerifyStep

    torch.cuda.set_device(local_rank)
    jsv.load()
    gb = GpuBench(local_rank)
    wl, tokens, g = load_workload(args.workload)
    st = VerifyStep(wl, tokens, device=gb.dev)
    model = workload_model(wl)
    stream = gb.stream

    if args.profile:
        if args.profile == "tree":
            call = tree_call(wl, st, gb.dev)
        elif args.profile == "qkv":
            call = qkv_rope_call(wl, st, gb.dev)
        else:
            call = getattr(st, args.profile)
        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            call()
        e1.record(stream)
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0
        eager_us = 1e3 * e0.elapsed_time(e1) / args.steps
        # the same calls from one CUDA graph: device time without host launch gaps
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(args.steps):
                call()
        graph.replay()
        torch.cuda.synchronize()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0
        gb.clocks.stop()
        print(json.dumps({"profile": args.profile, "workload": args.workload, "mean_us_warm_l2": eager_us,
                          "graph_us_warm_l2": 1e3 * e0.elapsed_time(e1) / args.steps}), flush=True)
        del graph
        return

    # correctness of this very launch configuration against stored oracle values
    st.run()
    torch.cuda.synchronize()
    check = check_against_golden(st, g)
    hist = accept_hist(st.accept_len.cpu().numpy())

    for _ in range(max(args.warmup, 3)):
        gb.flush_l2(1)
        st.run()
    torch.cuda.synchronize()

    K = args.steps
    # timed region 1 (the headline): exactly K whole steps, events around each
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = jsv.jsv_kernel_launches()
    steps = gb.time_steps(st.run, K, "steps")
    launches = jsv.jsv_kernel_launches() - launches0
    if world > 1:
        torch.distributed.barrier()
    stat = step_stats(steps)
    step_ms = stat["median"] * 1e-3
    assert int(st.status.item()) == 0

    # timed region 2: the same steps with an event between calls, for the
    # per-call durations (the dominant kernel's roofline uses these)
    per = gb.time_calls(st, K, "calls")
    call_ms = np.median(per, axis=0)
    assert int(st.status.item()) == 0

    # timed region 3: the same step replayed from one CUDA graph
    graph = None
    if not args.no_graph:
        st.capture()
        for _ in range(3):
            st.replay()
        torch.cuda.synchronize()
        graph = float(np.median(gb.time_steps(st.replay, K, "graph")))
        assert int(st.status.item()) == 0

    # tree construction (accum_logp) for this workload's tree shape, per request
    tree_us = None
    if not args.no_graph:
        build_tree = tree_call(wl, st, gb.dev)
        for _ in range(3):
            build_tree()
        torch.cuda.synchronize()
        tree_us = 1e3 * float(np.median(gb.time_steps(build_tree, K, "tree")))
        assert int(st.status.item()) == 0

    # tree Q/K/V projection + rotary + paged K/V append (the step before the attention)
    qkv = None
    if not args.no_graph:
        rows = (wl.Hq + 2 * wl.Hkv) * wl.D
        qkv_call = qkv_rope_call(wl, st, gb.dev)
        for _ in range(3):
            qkv_call()
        torch.cuda.synchronize()
        q_us = 1e3 * float(np.median(gb.time_steps(qkv_call, K, "qkv")))
        assert int(st.status.item()) == 0
        q_bytes = rows * wl.d * 2 + wl.T * wl.d * 2 + wl.T * rows * 2
        qkv = {"us_per_call": q_us, "algorithmic_bytes": q_bytes,
               "achieved_gbs": q_bytes / (q_us * 1e-6) / 1e9,
               "call": "jsv_tree_qkv_rope (the projection feeding the verify step; not timed in it)"}

    # end to end through the public API with host buffers: per step the input
    # copy up, the step, the output copy back and a host synchronisation,
    # timed by the host clock
    e2e = None
    if not args.no_e2e:
        h2d, d2h = st.h2d_bytes(), st.d2h_bytes()
        for _ in range(3):
            st.run_host()
            stream.synchronize()
        host_ms = []
        with gb.clocks.region("e2e"):
            for i in range(K):
                gb.flush_l2(i)
                torch.cuda.synchronize()
                t0 = time.perf_counter()
                out = st.run_host()
                stream.synchronize()
                host_ms.append((time.perf_counter() - t0) * 1e3)
        assert int(out["accept_len"][0]) == g["accept_len"][0]
        e2e_stat = step_stats(host_ms)
        e2e = {"ms": e2e_stat["median"] * 1e-3, "stat": e2e_stat,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        # the same end-to-end step from one CUDA graph (copies included)
        if not args.no_graph:
            st.capture_host()
            for _ in range(3):
                st.replay_host()
            stream.synchronize()
            host_ms = []
            with gb.clocks.region("e2e_graph"):
                for i in range(K):
                    gb.flush_l2(i)
                    torch.cuda.synchronize()
                    t0 = time.perf_counter()
                    out = st.replay_host()
                    stream.synchronize()
                    host_ms.append((time.perf_counter() - t0) * 1e3)
            assert int(out["accept_len"][0]) == g["accept_len"][0]
            e2e["graph_stat"] = step_stats(host_ms)

    # max over ranks
    e2e_graph_ms = e2e["graph_stat"]["median"] * 1e-3 if e2e and "graph_stat" in e2e else 0.0
    step_ms_max, e2e_ms_max, graph_ms_max, e2e_graph_ms_max = reduce_max_over_ranks(
        [step_ms, e2e["ms"] if e2e else 0.0, graph or 0.0, e2e_graph_ms], device=gb.dev)

    # the other workloads (one GPU only; replicas would repeat them)
    pk = peaks()
    extra = {}
    if world == 1 and args.workloads != "none":
        names = [n for n in DESCRIPTION if n != args.workload] if args.workloads == "all" else \
            [n for n in args.workloads.split(",") if n and n != args.workload]
        del st
        torch.cuda.empty_cache()
        for n in names:
            extra[n] = measure_workload(gb, n, max(50, K), args.warmup, pk)
    gb.clocks.stop()
    if rank != 0:
        return

    hbm, tf_burst, tf_sus, peak_kind = pk
    share = {n: float(call_ms[j] / call_ms.sum()) for j, n in enumerate(CALLS)}
    dom = "lmhead" if call_ms[1] >= call_ms[0] else "attention"
    dom_ms = float(call_ms[CALLS.index(dom)])
    m = model[dom]
    t_hbm = m["bytes"] / (hbm * 1e9)
    t_tc = m["flops"] / (tf_burst * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": m["bytes"] / (dom_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": m["flops"] / (dom_ms * 1e-3) / 1e12, "peak": tf_burst,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = {"lmhead": "jsv_lmhead_argmax", "attention": "jsv_tree_attention"}[dom]
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"
    roof["duration"] = "median of the per-call CUDA-event times over the timed steps"
    roof["algorithmic_bytes_per_launch"] = m["bytes"]
    roof["algorithmic_flops_per_launch"] = m["flops"]
    roof["traffic"] = ncu_traffic(dom, args.workload)

    value = whole_job_value(wl.T, world, step_ms_max)
    line = {
        "metric": METRIC, "value": value, "unit": "nodes/s", "n_gpus": world, "steps": K,
        "warmup": max(args.warmup, 3), "ms_per_step": step_ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": DESCRIPTION[args.workload], "name": args.workload,
                   "nodes_per_step": wl.T, "requests": wl.B,
                   "prefix_tokens": int(wl.prefix_len.sum()),
                   "l2": f"flushed before every timed step: a {gb.flush_bytes >> 20} MiB write (4x the "
                         f"device's {gb.l2_bytes >> 20} MiB L2), then a read of it, so the flush's own dirty "
                         f"lines are written back before the timed region",
                   "parallelism": f"replicas x{world}"},
        "step_latency_us": step_ms_max * 1e3,
        "step_us": stat,
        "statistic": "median of the timed steps (p10/p90/mean in step_us)",
        **fractions(model, step_ms_max * 1e3, hbm, tf_burst, tf_sus),
        "step_hbm_bytes": model["step_hbm_bytes"],
        "call_us": {n: float(call_ms[j] * 1e3) for j, n in enumerate(CALLS)},
        "call_share": share,
        "call_sum_us": float(call_ms.sum() * 1e3),
        "roofline": roof,
        "gpu_launches": int(launches),
        "clocks": gb.clocks.summary(["steps", "calls", "graph"]),
        "clocks_all_regions": gb.clocks.summary(),
        "check": check,
        "accept_len_hist": hist, "tokens_per_forward_mean": tpf_mean(hist),
    }
    if qkv is not None:
        qkv["frac_of_hbm_peak"] = qkv["achieved_gbs"] / hbm
        line["qkv_rope"] = qkv
    if tree_us is not None:
        Dt, kt, bt = TREE_SHAPE[args.workload]
        line["tree_build"] = {"us_per_call": tree_us, "requests": wl.B, "depth": Dt, "width": kt, "budget": bt,
                              "call": "jsv_accum_logp_tree (not part of the verify step)"}
    if graph:
        line["graph"] = {"value": whole_job_value(wl.T, world, graph_ms_max), "unit": "nodes/s",
                         "ms_per_step": graph_ms_max,
                         "how": "the step's calls captured once in a CUDA graph, replayed per step (median)"}
    if e2e:
        eager = {"value": whole_job_value(wl.T, world, e2e_ms_max), "unit": "nodes/s",
                 "ms_per_step": e2e_ms_max, "step_us": e2e["stat"],
                 "how": "VerifyStep.run_host: per step the input copy up (pinned), the calls from Python, "
                        "the output copy back and a stream synchronisation, host clock (median)"}
        if e2e_graph_ms_max > 0:
            # the engine form: the same copies and calls replayed from one CUDA graph
            line["e2e"] = {"value": whole_job_value(wl.T, world, e2e_graph_ms_max), "unit": "nodes/s",
                           "ms_per_step": e2e_graph_ms_max, "step_us": e2e["graph_stat"],
                           "how": "VerifyStep.replay_host: per step one replay of a CUDA graph holding the input "
                                  "copy up (pinned), the calls and the output copy back, then a stream "
                                  "synchronisation, host clock (median)",
                           "eager": eager}
        else:
            line["e2e"] = dict(eager)
        line["e2e"]["h2d_bytes_per_step"] = e2e["h2d_bytes_per_step"]
        line["e2e"]["d2h_bytes_per_step"] = e2e["d2h_bytes_per_step"]
    if extra:
        line["workloads"] = extra
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, tokens, g)
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        # a short timeout, so that the ranks still waiting end with an error if
        # one rank fails (tests/test_multirank.py shows it with gloo); it is
        # well above the longest stretch between two collectives here
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    try:
        run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
