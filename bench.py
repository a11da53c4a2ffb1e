#!/usr/bin/env python
"""Benchmark of the packed-tree SSM scan + commit on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
build the tree masks once, then the fused scan + commit of every layer (y for
every node, h_new for the accepted path).  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config m2_2p7b]
    python bench.py --impl reference ...      # the CPU oracle arm

Timing: CUDA events on the launching stream, K steps bracketed by a barrier and
a synchronize, max over ranks.  Workloads smaller than L2 rotate over enough
copies of their buffers that each step reads data that is not L2-resident.
Multi-GPU (torchrun): every rank runs its own batch (weak scaling); the path has
no exchange step, so no collective touches the data.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tree-scan nodes/sec and achieved HBM GB/s (% of roofline), 1×B200"
UNIT = "nodes/s"
DEFAULT_CONFIG = "m2_2p7b"
# Extra workloads that also get an end-to-end figure, and that also run the
# unrolled baseline and the verification timing (the wide trees would need tens
# of GB of per-path states unrolled).
E2E_WORKLOADS = ("serve64",)
SIDE_WORKLOADS = ("m2_2p7b", "hyb8b", "serve64")
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--kernel", choices=["auto", "simt", "tc", "small"], default="auto")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle sample budget")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling)")
    ap.add_argument("--layers", type=int, default=None, help="override the workload's layer count (profiling)")
    ap.add_argument("--also", default="tiny,hyb8b,serve64,wide256,wide256_chain",
                    help="comma-separated extra workloads summarised in the same line ('none' to skip)")
    ap.add_argument("--no-separate", action="store_true",
                    help="skip the stand-alone scan and commit timings")
    ap.add_argument("--no-unrolled", action="store_true",
                    help="skip the unrolled-tree baseline comparison (one layer per workload)")
    ap.add_argument("--no-accept", action="store_true",
                    help="skip the greedy tree-verification timing (argmax over the logits + walk)")
    ap.add_argument("--no-floor", action="store_true", help="skip the launch and state-copy latency floors")
    ap.add_argument("--no-attention", action="store_true",
                    help="skip the tree-masked attention timing (the hybrid's Transformer layers)")
    ap.add_argument("--no-gdn", action="store_true",
                    help="skip the gated-delta-rule tree timing (linear-attention layers)")
    ap.add_argument("--vocab", type=int, default=50280,
                    help="vocabulary of the synthetic logits for the verification timing (Mamba2-2.7B's padded vocab)")
    return ap.parse_args()


def default_steps(name):
    return {"tiny": 200, "m2_2p7b": 400, "m2_2p7b_16": 400, "hyb8b": 200,
            "serve64": 30, "wide256": 30, "wide256_chain": 20}.get(name, 50)


# ----------------------------------------------------------------------------- accounting


def algorithmic_bytes(w):
    """Bytes of one fused scan + commit launch (one layer): every tensor moved once."""
    b, T, H, P, N, G = w.batch, w.n_nodes, w.nheads, w.headdim, w.dstate, w.ngroups
    e = 2 if w.dtype == "bf16" else 4
    state = b * H * P * N * 4
    xy = b * T * H * P * e
    return {
        "h0": state, "h_new": state, "x": xy, "y": xy, "dt": b * T * H * e,
        "B": b * T * G * N * e, "C": b * T * G * N * e, "A": H * 4, "D": H * 4,
        "parent": b * T * 4, "path": b * w.maxlen * 4 + b * 4,
    }


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_sha(fname):
    import hashlib
    src = os.path.join(ROOT, "hybrid_packed_tree_b200", "csrc", fname)
    return hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] if os.path.exists(src) else None


def profile_traffic(kernel_name, workload):
    """Per-launch DRAM bytes (read + write) of a kernel on this workload, from the
    committed ncu figures (profiles/traffic.json), if they were taken on the current
    kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        entries = json.load(f).get("entries", [])
    for e in entries:
        if e.get("kernel") != kernel_name or e.get("workload") != workload:
            continue
        if source_sha(e.get("file", "")) != e.get("sha"):
            return None
        return float(e["bytes_per_launch"])
    return None


KERNEL_NAMES = {"small": "scan_small_kernel", "tc": "scan_tc_kernel", "simt": "scan_simt_kernel"}


def commit_bytes(w):
    """Bytes of one stand-alone commit launch (one layer): h0 read, h_new written,
    the path, and x, dt and B at the accepted path's nodes."""
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    e = 2 if w.dtype == "bf16" else 4
    nodes = int(np.sum(w.path_len))
    return 2 * b * H * P * N * 4 + b * w.maxlen * 4 + b * 4 + nodes * (H * P * e + H * e + G * N * e)


def scan_bytes(w):
    """Bytes of one stand-alone scan launch (one layer): every input once and y."""
    a = algorithmic_bytes(w)
    return sum(v for k, v in a.items() if k not in ("h_new", "path"))


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.strip().split(",") for r in self.file.read().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                for nm, v in zip(names, r[5:9]):
                    if "Active" in v and "Not" not in v:
                        reasons.add(nm)
            except Exception:
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- ranks


def max_over_ranks(values, world, device):
    """Each timing becomes its maximum over the ranks (identity on one rank)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_scaling_value(units_per_rank_step, steps, ms, world):
    """Whole-job throughput: every rank processes its own batch, time is the slowest rank's."""
    return world * units_per_rank_step * steps / (ms / 1e3)


# ----------------------------------------------------------------------------- our arm


def workload_config(name, batch=None, layers=None):
    """The workload keys of the JSON line's `config` (the same for both arms)."""
    from hybrid_packed_tree_b200 import workloads as wl
    _, b0, l0, H, P, N, G, T, io, _ = wl.SPECS[name]
    return {"workload": name, "batch": batch or b0, "layers": layers or l0, "n_nodes": T, "nheads": H,
            "headdim": P, "dstate": N, "ngroups": G, "io_dtype": io, "state_dtype": "f32"}


def dev_tensor(torch, a, io, device):
    if io == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def run_unrolled(name, local_rank, steps=5):
    """The unrolled-tree baseline on one layer of a workload: every root-to-leaf path
    scanned as its own sequence with its own state (stree_unrolled_scan), timed as a
    CUDA graph of `steps` launches after an L2 flush."""
    import torch

    from hybrid_packed_tree_b200 import stree
    from hybrid_packed_tree_b200 import workloads as wl

    device = torch.device("cuda", local_rank)
    w = wl.make_workload(name, layers=1)
    paths, plen = wl.unroll_paths(w.parent)
    L, io = w.layers[0], w.dtype
    d = {k: dev_tensor(torch, getattr(L, k), io, device) for k in ("x", "dt", "B", "C")}
    d.update({k: dev_tensor(torch, getattr(L, k), "f32", device) for k in ("A", "D", "h0")})
    pt, lt = torch.from_numpy(paths).to(device), torch.from_numpy(plen).to(device)
    b, n_paths, depth = paths.shape
    y = torch.empty((b, n_paths, depth, w.nheads, w.headdim), dtype=d["x"].dtype, device=device)
    h = torch.empty((b, n_paths, w.nheads, w.headdim, w.dstate), dtype=torch.float32, device=device)
    err = torch.zeros(4, dtype=torch.int32, device=device)

    def call():
        stree.stree_unrolled_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"], pt, lt, y, h,
                                  err_out=err, stream=torch.cuda.current_stream(device))

    for _ in range(3):
        call()
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(steps):
            call()
    g.replay()
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(int(3 * l2) // 4 + 1, dtype=torch.float32, device=device)
    flush.zero_()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    g.replay()
    t1.record()
    torch.cuda.synchronize(device)
    if int(err[0]) != 0:
        raise RuntimeError(f"device error in the unrolled baseline: {err.tolist()}")
    ms = t0.elapsed_time(t1) / steps
    del g
    state = w.nheads * w.headdim * w.dstate * 4
    real = int((plen > 0).sum())
    return {"workload": name, "layers": 1, "ms_per_launch": ms, "paths": real, "path_positions": int(plen.sum()),
            "tree_nodes": w.batch * w.n_nodes, "path_state_bytes": real * state,
            "nodes_per_s": w.batch * w.n_nodes / (ms / 1e3)}


def run_accept(name, vocab, local_rank, steps=20):
    """Greedy tree verification (stree_accept_greedy) on synthetic bf16 logits
    [b, T, vocab] of a workload's trees, timed as a CUDA graph of `steps` calls after
    an L2 flush.  Its bytes are the logits (argmax) plus the small tree inputs."""
    import torch

    from hybrid_packed_tree_b200 import stree
    from hybrid_packed_tree_b200 import workloads as wl

    device = torch.device("cuda", local_rank)
    w = wl.make_workload(name, layers=1)
    b, T = w.batch, w.n_nodes
    gen = torch.Generator(device=device)
    gen.manual_seed(1234)
    # Distinct logits per call (up to `steps` copies, enough that no call finds its
    # logits in L2 after the flush).
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nsets = max(1, min(steps, -(-3 * l2 // (b * T * vocab * 2))))
    logit_sets = [torch.randn((b, T, vocab), generator=gen, device=device).to(torch.bfloat16) for _ in range(nsets)]
    tokens = torch.randint(0, vocab, (b, T), generator=gen, device=device, dtype=torch.int32)
    parent = torch.from_numpy(w.parent).to(device)
    pred = torch.empty((b, T), dtype=torch.int32, device=device)
    path = torch.empty((b, T), dtype=torch.int32, device=device)
    plen = torch.empty((b,), dtype=torch.int32, device=device)
    bonus = torch.empty((b,), dtype=torch.int32, device=device)
    err = torch.zeros(4, dtype=torch.int32, device=device)

    def call(i):
        stree.stree_accept_greedy(logit_sets[i % nsets], tokens, parent, pred, path, plen, bonus, err_out=err,
                                  stream=torch.cuda.current_stream(device))

    for i in range(3):
        call(i)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            call(i)
    g.replay()
    flush = torch.empty(int(3 * l2) // 4 + 1, dtype=torch.float32, device=device)
    flush.zero_()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    g.replay()
    t1.record()
    torch.cuda.synchronize(device)
    if int(err[0]) != 0:
        raise RuntimeError(f"device error in the verification step: {err.tolist()}")
    ms = t0.elapsed_time(t1) / steps
    del g
    nbytes = b * T * vocab * 2 + b * T * 4 * 3 + b * T * 4 + b * 8
    hbm_gbs, peak_kind = peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": name, "vocab": vocab, "logits_dtype": "bf16", "ms_per_call": ms, "bytes_per_call": nbytes,
            "achieved_gbs": gbs, "frac": gbs / hbm_gbs, "peak_source": f"{peak_kind} hbm_gbs",
            "timing": f"{steps} calls in one CUDA graph after an L2 flush, {nsets} distinct logits buffers"}


def gdn_bytes(b, T, Hv, Hk, dk, dv, e, maxlen, nodes_on_paths):
    """Bytes of one gated-delta-rule tree call with commit: S0 read and S_new
    written (fp32), q, k, v, o, the gates, the tree and the paths."""
    return (2 * b * Hv * dv * dk * 4 + 2 * b * T * Hk * dk * e + 2 * b * T * Hv * dv * e + 2 * b * T * Hv * 4
            + b * T * 4 + b * maxlen * 4 + b * 4)


def run_gdn(name, local_rank, steps=50, heads_v=32, heads_k=16, linear=False):
    """The gated delta rule over a workload's trees (one linear-attention layer:
    32 value heads, 16 query/key heads, d_k = d_v = 128, bf16 inputs, fp32 state),
    fused with the commit of the workload's accepted paths; a CUDA graph of `steps`
    calls over rotated buffers after an L2 flush.  linear=True: zero erase strength
    (gated linear attention; the erase array adds its bytes)."""
    import torch

    from hybrid_packed_tree_b200 import stree
    from hybrid_packed_tree_b200 import workloads as wl

    device = torch.device("cuda", local_rank)
    w = wl.make_workload(name, layers=1)
    g = wl.gdn_inputs(w.parent, w.path, w.path_len, heads_v=heads_v, heads_k=heads_k, dtype="bf16", seed=41)
    b, T = w.parent.shape
    nbytes = gdn_bytes(b, T, heads_v, heads_k, 128, 128, 2, w.maxlen, int(np.sum(w.path_len)))
    if linear:
        nbytes += b * T * heads_v * 4
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nsets = max(1, -(-3 * l2 // nbytes))
    sets = []
    for _ in range(nsets):
        d = {k: dev_tensor(torch, getattr(g, k), "bf16", device) for k in ("q", "k", "v")}
        d.update({k: dev_tensor(torch, getattr(g, k), "f32", device) for k in ("alpha", "beta", "S0")})
        d.update({k: torch.from_numpy(np.ascontiguousarray(getattr(g, k))).to(device)
                  for k in ("parent", "path", "path_len")})
        d["o"] = torch.empty_like(d["v"])
        d["S_new"] = torch.empty_like(d["S0"])
        d["erase"] = torch.zeros_like(d["beta"]) if linear else None
        sets.append(d)
    err = torch.zeros(4, dtype=torch.int32, device=device)

    def call(i):
        d = sets[i % nsets]
        stree.stree_gdn_tree_scan_commit(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["S0"], d["parent"],
                                         d["o"], d["path"], d["path_len"], d["S_new"], err_out=err,
                                         stream=torch.cuda.current_stream(device), erase=d["erase"])

    for i in range(3):
        call(i)
    torch.cuda.synchronize(device)
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for i in range(steps):
            call(i)
    gr.replay()
    flush = torch.empty(int(3 * l2) // 4 + 1, dtype=torch.float32, device=device)
    flush.zero_()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    gr.replay()
    t1.record()
    torch.cuda.synchronize(device)
    if int(err[0]) != 0:
        raise RuntimeError(f"device error in the gated-delta-rule step: {err.tolist()}")
    ms = t0.elapsed_time(t1) / steps
    del gr
    hbm_gbs, peak_kind = peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    rule = "gated linear attention (zero erase)" if linear else "gated delta rule"
    return {"workload": f"{name} trees, {rule} ({heads_v} value / {heads_k} key heads, d_k = d_v = 128)",
            "batch": b, "n_nodes": T, "ms_per_call": ms, "nodes_per_s": b * T / (ms / 1e3),
            "bytes_per_call": nbytes, "achieved_gbs": gbs, "frac": gbs / hbm_gbs,
            "peak_source": f"{peak_kind} hbm_gbs",
            # bf16, d = 128, up to 64 nodes: the tensor-core kernel; else the CUDA-core one
            "kernel": "gdn_tc_kernel" if T <= 64 else "gdn_tree_kernel",
            "timing": f"{steps} calls in one CUDA graph after an L2 flush, {nsets} rotated buffer sets"}


def run_sampling(name, vocab, local_rank, steps=20, temperature=1.0):
    """Stochastic tree verification (stree_accept_sampling) on synthetic target and
    draft logits [b, T, vocab] (bf16) of a workload's trees, timed as a CUDA graph of
    `steps` calls after an L2 flush.  Its algorithmic bytes are the logits rows of
    the nodes the walks visit (target and draft; the residual passes re-read a draft
    row from L2), counted from the returned paths."""
    import torch

    from hybrid_packed_tree_b200 import stree
    from hybrid_packed_tree_b200 import workloads as wl

    device = torch.device("cuda", local_rank)
    w = wl.make_workload(name, layers=1)
    b, T = w.parent.shape
    tl, dl, tokens, ua, ub = wl.sampling_inputs(w.parent, vocab, seed=21, dtype="bf16")
    t_logits = [dev_tensor(torch, tl, "bf16", device)]
    d_logits = [dev_tensor(torch, dl, "bf16", device)]
    tok = torch.from_numpy(tokens).to(device)
    par = torch.from_numpy(w.parent).to(device)
    uat = torch.from_numpy(ua).to(device)
    ubt = torch.from_numpy(ub).to(device)
    path = torch.empty((b, T), dtype=torch.int32, device=device)
    plen = torch.empty((b,), dtype=torch.int32, device=device)
    bonus = torch.empty((b,), dtype=torch.int32, device=device)
    err = torch.zeros(4, dtype=torch.int32, device=device)

    def call(i):
        stree.stree_accept_sampling(t_logits[i % len(t_logits)], d_logits[i % len(d_logits)], tok, par, temperature,
                                    uat, ubt, path, plen, bonus, err_out=err, stream=torch.cuda.current_stream(device))

    call(0)
    torch.cuda.synchronize(device)
    # Copies of the logits (same values, so the same walks) rotated so that the
    # rows a call visits are not left in L2 by the calls before it.
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    visited = int(plen.sum().item())
    nsets = max(1, min(steps, -(-3 * l2 // max(1, 2 * visited * vocab * 2))))
    while len(t_logits) < nsets:
        t_logits.append(t_logits[0].clone())
        d_logits.append(d_logits[0].clone())
    for i in range(3):
        call(i)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            call(i)
    g.replay()
    flush = torch.empty(int(3 * l2) // 4 + 1, dtype=torch.float32, device=device)
    flush.zero_()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    g.replay()
    t1.record()
    torch.cuda.synchronize(device)
    if int(err[0]) != 0:
        raise RuntimeError(f"device error in the sampling verification: {err.tolist()}")
    ms = t0.elapsed_time(t1) / steps
    del g
    nbytes = 2 * visited * vocab * 2
    hbm_gbs, peak_kind = peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"workload": name, "vocab": vocab, "logits_dtype": "bf16", "temperature": temperature,
            "ms_per_call": ms, "accepted_nodes": visited, "bytes_per_call": nbytes, "achieved_gbs": gbs,
            "frac": gbs / hbm_gbs, "peak_source": f"{peak_kind} hbm_gbs",
            "timing": f"{steps} calls in one CUDA graph after an L2 flush, {nsets} rotated copies of the logits"}


def run_floor(name, local_rank, steps=200):
    """Latency floors of one step on this GPU, for comparison with the scan's step
    time: a CUDA graph of `steps` launches of a one-element kernel (launch and
    completion only), and of copies of the workload's state (h0 -> h_new, the
    dominant bytes of the fused step) over rotated buffers after an L2 flush."""
    import torch

    from hybrid_packed_tree_b200 import workloads as wl

    device = torch.device("cuda", local_rank)
    w = wl.make_workload(name, layers=1)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    state = w.batch * w.nheads * w.headdim * w.dstate
    nsets = max(1, -(-3 * l2 // (8 * state)))
    src = [torch.randn(state, device=device) for _ in range(nsets)]
    dst = [torch.empty_like(x) for x in src]
    one = torch.zeros(1, device=device)

    def timed(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(steps):
                fn(i)
        g.replay()
        flush = torch.empty(int(3 * l2) // 4 + 1, dtype=torch.float32, device=device)
        flush.zero_()
        torch.cuda.synchronize(device)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        g.replay()
        t1.record()
        torch.cuda.synchronize(device)
        del g
        return t0.elapsed_time(t1) / steps * 1e3

    empty_us = timed(lambda i: one.add_(1.0))
    copy_us = timed(lambda i: dst[i % nsets].copy_(src[i % nsets]))
    return {"workload": name, "empty_kernel_us": empty_us, "state_copy_us": copy_us,
            "state_copy_bytes": 8 * state,
            "note": "CUDA graphs of back-to-back launches: a one-element torch kernel, and a torch copy of the "
                    "workload's fp32 state (read + write) over rotated buffers"}


ATTN_CTX = {"hyb8b": 4096, "serve64": 1024}


def run_attention(name, local_rank, steps=20, heads_q=32, heads_kv=8):
    """Tree-masked attention over a workload's trees (one attention layer of a
    hybrid model: 32 query heads, 8 key/value heads, head dim 128, bf16), every
    sequence with a full context of ATTN_CTX[name] cached tokens; a CUDA graph of
    `steps` calls over rotated buffers after an L2 flush.  Reports HBM bytes (the
    context keys and values, the tree's, q and o) and the tensor flops actually
    issued (two 128-row products per key block and query tile)."""
    import torch

    from hybrid_packed_tree_b200 import stree
    from hybrid_packed_tree_b200 import workloads as wl

    device = torch.device("cuda", local_rank)
    w = wl.make_workload(name, layers=1)
    b, T = w.parent.shape
    S = ATTN_CTX.get(name, 2048)
    a = wl.attention_inputs(w.parent, S, [S] * b, heads_q=heads_q, heads_kv=heads_kv, seed=71, stale=0.0)
    d = 128
    nbytes = 2 * b * S * heads_kv * d * 2 + 2 * b * T * heads_kv * d * 2 + 2 * b * T * heads_q * d * 2 + b * T * 4
    G = heads_q // heads_kv
    tq = 128 // G
    tiles = b * heads_kv * (-(-T // tq))
    flops = tiles * 4 * 128 * 128 * d * (-(-S // 128) + 1)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nsets = max(1, -(-3 * l2 // nbytes))

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)

    base = {k: bf(a[k]) for k in ("q", "k_ctx", "v_ctx", "k_tree", "v_tree")}
    sets = [base] + [{k: v.clone() for k, v in base.items()} for _ in range(nsets - 1)]
    ctx_len = torch.from_numpy(a["ctx_len"]).to(device)
    parent = torch.from_numpy(a["parent"]).to(device)
    outs = [torch.empty_like(base["q"]) for _ in range(nsets)]
    err = torch.zeros(4, dtype=torch.int32, device=device)
    ws_bytes = stree.stree_tree_attention_workspace_size(T, b, S, heads_q, heads_kv, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device) if ws_bytes else None

    def call(i):
        t = sets[i % nsets]
        stree.stree_tree_attention(t["q"], t["k_ctx"], t["v_ctx"], t["k_tree"], t["v_tree"], ctx_len, parent,
                                   outs[i % nsets], a["scale"], err, workspace=ws,
                                   stream=torch.cuda.current_stream(device))

    for i in range(3):
        call(i)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(steps):
            call(i)
    g.replay()
    flush = torch.empty(int(3 * l2) // 4 + 1, dtype=torch.float32, device=device)
    flush.zero_()
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    g.replay()
    t1.record()
    torch.cuda.synchronize(device)
    if int(err[0]) != 0:
        raise RuntimeError(f"device error in the tree attention: {err.tolist()}")
    ms = t0.elapsed_time(t1) / steps
    del g
    hbm_gbs, peak_kind = peaks()
    tflops_peak = measured_tflops()
    gbs = nbytes / (ms / 1e3) / 1e9
    tfs = flops / (ms / 1e3) / 1e12
    return {"workload": f"{name} trees, {S} cached tokens per sequence", "batch": b, "n_nodes": T,
            "heads_q": heads_q, "heads_kv": heads_kv, "head_dim": d, "ms_per_call": ms,
            "bytes_per_call": nbytes, "achieved_gbs": gbs, "frac_hbm": gbs / hbm_gbs,
            "tensor_flops_per_call": flops, "achieved_tflops": tfs,
            "frac_tensor": tfs / tflops_peak if tflops_peak else None, "kernel": "tree_attention_kernel",
            "workspace_bytes": ws_bytes,
            "peak_source": f"{peak_kind} hbm_gbs, measured bf16_tflops",
            "timing": f"{steps} calls in one CUDA graph after an L2 flush, {nsets} rotated buffer sets"}


def measured_tflops():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


def unrolled_summary(o, u):
    """Unrolled baseline beside the packed scan (per layer: the packed step time
    divided by the layers)."""
    packed_ms = o["ms_per_step"] / o["config"]["layers"]
    u = dict(u)
    u["packed_ms_per_layer"] = packed_ms
    u["unrolled_over_packed_time"] = u["ms_per_launch"] / packed_ms
    return u


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from hybrid_packed_tree_b200 import stree
    from hybrid_packed_tree_b200 import workloads as wl

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    w = wl.make_workload(args.config, batch=args.batch, layers=args.layers)
    K = args.steps or default_steps(args.config)
    Wm = max(3, args.warmup)
    nl = w.nlayers
    io = w.dtype

    per_launch = algorithmic_bytes(w)
    launch_bytes = sum(per_launch.values())
    step_bytes = launch_bytes * nl
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nsets = max(1, -(-3 * l2 // step_bytes))          # rotated copies: > 3x L2 per cycle

    # Device buffers: nsets copies of every layer's inputs and outputs.
    sets = []
    for s in range(nsets):
        layers = []
        for li in range(nl):
            L = w.layers[li]
            d = {k: dev_tensor(torch, getattr(L, k), io, device) for k in ("x", "dt", "B", "C")}
            d.update({k: dev_tensor(torch, getattr(L, k), "f32", device) for k in ("A", "D", "h0")})
            d["y"] = torch.empty_like(d["x"])
            d["h_new"] = torch.empty_like(d["h0"])
            layers.append(d)
        tree = {"parent": torch.from_numpy(w.parent).to(device), "path": torch.from_numpy(w.path).to(device),
                "path_len": torch.from_numpy(w.path_len).to(device)}
        sets.append((layers, tree))

    ctx = stree.stree_ctx_create()
    stree.stree_ctx_set_kernel(ctx, args.kernel)
    stream = torch.cuda.current_stream(device)

    def step(i, ev=None):
        layers, tree = sets[i % nsets]
        s = torch.cuda.current_stream(device)          # the capture stream inside a graph
        # The first layer's call builds the step's tree; the other layers reuse it.
        for li, d in enumerate(layers):
            if ev is not None:
                ev[li][0].record(s)
            stree.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"],
                                         tree["parent"] if li == 0 else None, tree["path"], tree["path_len"],
                                         d["y"], d["h_new"], stream=s)
            if ev is not None:
                ev[li][1].record(s)

    for i in range(Wm):
        step(i)
    stree.stree_sync_check(ctx, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    # The K steps are captured once into a CUDA graph and replayed: the timed
    # region holds exactly the steps' kernels, back to back, with no host
    # launch overhead between them.  Launches are counted while capturing.
    n0 = stree.stree_ctx_launch_count(ctx)
    g_steps = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_steps):
        for i in range(K):
            step(i)
    launches = stree.stree_ctx_launch_count(ctx) - n0
    # A second graph of the same steps with timing events around every fused
    # call (the dominant kernel's launch duration for the roofline).
    evs = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(nl)]
           for _ in range(K)]
    g_events = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_events):
        for i in range(K):
            step(i, evs[i])
    for g in (g_steps, g_events):                      # one untimed replay each
        g.replay()
    # Written before each timed replay so that no step input starts in L2.
    flush = torch.empty(int(3 * l2) // 4 + 1, dtype=torch.float32, device=device)
    torch.cuda.synchronize(device)

    # Timed region 1: the step time (value).
    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    barrier()
    flush.zero_()
    torch.cuda.synchronize(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    g_steps.replay()
    t1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    ms = t0.elapsed_time(t1)

    # Timed region 2: per-launch durations.
    barrier()
    flush.zero_()
    torch.cuda.synchronize(device)
    g_events.replay()
    torch.cuda.synchronize(device)
    barrier()
    clk = clocks.stop()
    kern_ms = [e[0].elapsed_time(e[1]) for per in evs for e in per]
    del g_steps, g_events
    kernel_used = stree.stree_ctx_last_kernel(ctx)
    sep = None
    if not args.no_separate:
        sep = run_separate(torch, stree, w, ctx, sets, nsets, K, device, flush)
    del flush
    st, info = stree.stree_sync_check(ctx, stream, raise_on_error=False)
    if st != 0:
        raise RuntimeError(f"device error during the benchmark: {info}")

    ms, kmean = max_over_ranks([ms, statistics.mean(kern_ms)], world, device)
    if sep is not None:
        sep["scan"]["ms_per_launch"], sep["commit"]["ms_per_launch"] = max_over_ranks(
            [sep["scan"]["ms_per_launch"], sep["commit"]["ms_per_launch"]], world, device)
        hbm_gbs0, _ = peaks()
        for part in (sep["scan"], sep["commit"]):
            part["achieved_gbs"] = part["bytes_per_launch"] / (part["ms_per_launch"] / 1e3) / 1e9
            part["frac"] = part["achieved_gbs"] / hbm_gbs0

    nodes_step = w.batch * w.n_nodes * nl
    value = weak_scaling_value(nodes_step, K, ms, world)
    hbm_gbs, peak_kind = peaks()
    kernel_name = KERNEL_NAMES.get(kernel_used, kernel_used)
    step_gbs = step_bytes * K / (ms / 1e3) / 1e9
    # The kernel's average launch duration: when the step graph holds nothing but
    # one launch of it per layer, the timed region over the launch count; else the
    # mean of the event pairs around every launch (those event nodes also end the
    # overlap of consecutive launches, so they read a little high).
    only_scan = int(launches) == K * nl
    launch_ms = ms / (K * nl) if only_scan else kmean
    achieved = launch_bytes / (launch_ms / 1e3) / 1e9
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": Wm,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if io == "bf16" else "f32", "data": "synthetic (seeded; shapes and distributions of the workload)",
        "config": {
            **workload_config(args.config, args.batch, args.layers),
            "kernel": args.kernel, "parallelism": f"replicas x{world}",
            "l2": (f"rotates {nsets} buffer copies ({nsets * step_bytes / 2**20:.0f} MiB > 3x L2)"
                   if nsets > 1 else "step bytes exceed L2 (no reuse between steps)")
                  + "; 3x-L2 buffer written before each timed replay",
            "timing": "CUDA graph of the K steps, replayed once (CUDA events around the replay)",
        },
        "hbm": {"step_bytes": step_bytes, "gbs_step": step_gbs},
        "sequences_per_s": world * w.batch * K / (ms / 1e3),
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
            "frac": achieved / hbm_gbs, "traffic": profile_traffic(kernel_name, args.config),
            "peak_source": f"{peak_kind} hbm_gbs", "kernel": kernel_name,
            "bytes_per_launch": launch_bytes, "kernel_ms_mean": launch_ms,
            "launch_ms_from": "step graph / launches" if only_scan else "events around every launch",
            "kernel_ms_events": kmean, "kernel_ms_events_median": statistics.median(kern_ms),
            "achieved_events": launch_bytes / (kmean / 1e3) / 1e9,
            "frac_events": launch_bytes / (kmean / 1e3) / 1e9 / hbm_gbs,
        },
        "clocks": clk,
        "gpu_launches": int(launches),
    }
    if sep is not None:
        out["separate"] = sep

    if not args.no_e2e:
        out["e2e"] = e2e(torch, stree, w, ctx, device, stream, args, world)
    stree.stree_ctx_destroy(ctx)
    return out


def run_separate(torch, stree, w, ctx, sets, nsets, K, device, flush):
    """The stand-alone scan (stree_tree_scan) and commit (stree_commit) of every layer,
    each call bracketed by timing events inside one CUDA graph of K steps, replayed
    after an L2 flush.  Returns per-launch means and the algorithmic bytes of each."""
    nl = w.nlayers
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(K * nl)]

    def step(i):
        layers, tree = sets[i % nsets]
        s = torch.cuda.current_stream(device)
        for li, d in enumerate(layers):
            e = ev[i * nl + li]
            e[0].record(s)
            stree.stree_tree_scan(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"],
                                  tree["parent"] if li == 0 else None, d["y"], stream=s)
            e[1].record(s)
            e[2].record(s)
            stree.stree_commit(ctx, tree["path"], tree["path_len"], d["h_new"], stream=s)
            e[3].record(s)

    step(0)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(K):
            step(i)
    g.replay()
    flush.zero_()
    torch.cuda.synchronize(device)
    g.replay()
    torch.cuda.synchronize(device)
    scan_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    commit_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
    kernel_used = stree.stree_ctx_last_kernel(ctx)
    del g
    return {
        "scan": {"kernel": KERNEL_NAMES.get(kernel_used, kernel_used), "ms_per_launch": scan_ms,
                 "bytes_per_launch": scan_bytes(w)},
        "commit": {"kernel": "commit_prep_kernel + " + ("commit_stream128_kernel" if w.dstate == 128 and w.headdim >= 64
                                                         else "commit_stream_kernel"),
                   "ms_per_launch": commit_ms, "bytes_per_launch": commit_bytes(w)},
        "timing": f"{K} steps x {nl} layers of scan-then-commit in one CUDA graph after an L2 flush, "
                  "timing events around every call",
    }


def e2e(torch, stree, w, ctx, device, stream, args, world):
    """Same metric through the public API with pinned host buffers: H2D of every
    input of the step, the calls, D2H of y and h_new, all inside the timed region."""
    import torch.distributed as dist
    io = w.dtype
    host_layers = []
    for L in w.layers:
        hl = {}
        for k in ("x", "dt", "B", "C", "A", "D", "h0"):
            t = dev_tensor(torch, getattr(L, k), io if k in ("x", "dt", "B", "C") else "f32", "cpu")
            hl[k] = t.pin_memory()
        hl["y"] = torch.empty_like(hl["x"]).pin_memory()
        hl["h_new"] = torch.empty_like(hl["h0"]).pin_memory()
        host_layers.append(hl)
    htree = {k: torch.from_numpy(getattr(w, k)).pin_memory() for k in ("parent", "path", "path_len")}
    dl = [{k: torch.empty_like(v, device=device) for k, v in hl.items()} for hl in host_layers]
    dtree = {k: torch.empty_like(v, device=device) for k, v in htree.items()}
    h2d = sum(v.numel() * v.element_size() for hl in host_layers for k, v in hl.items() if k not in ("y", "h_new"))
    h2d += sum(v.numel() * v.element_size() for v in htree.values())
    d2h = sum(hl[k].numel() * hl[k].element_size() for hl in host_layers for k in ("y", "h_new"))

    def step():
        for k in dtree:
            dtree[k].copy_(htree[k], non_blocking=True)
        for li, (hl, d) in enumerate(zip(host_layers, dl)):
            for k in ("x", "dt", "B", "C", "A", "D", "h0"):
                d[k].copy_(hl[k], non_blocking=True)
            stree.stree_tree_scan_commit(ctx, d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["h0"],
                                         dtree["parent"] if li == 0 else None, dtree["path"], dtree["path_len"],
                                         d["y"], d["h_new"], stream=stream)
            hl["y"].copy_(d["y"], non_blocking=True)
            hl["h_new"].copy_(d["h_new"], non_blocking=True)

    K = max(3, min(args.steps or default_steps(args.config), 50 if w.nlayers * w.batch < 64 else 5))
    for _ in range(3):
        step()
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    ms = t0.elapsed_time(t1)
    (ms,) = max_over_ranks([ms], world, device)
    nodes = w.batch * w.n_nodes * w.nlayers
    return {"value": weak_scaling_value(nodes, K, ms, world), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": K}


# ----------------------------------------------------------------------------- oracle arm


def oracle_sample(name):
    """A bounded sample of the workload for the CPU oracle: its first layer and at
    most 8 sequences.  Returns (workload, description)."""
    from hybrid_packed_tree_b200 import workloads as wl
    b0 = wl.SPECS[name][1]
    nb = min(b0, 8 if name not in ("wide256", "wide256_chain") else 2)
    w = wl.make_workload(name, batch=nb, layers=1)
    return w, f"layer 0 of {name}, {nb} of {b0} sequence(s), full heads and tree; scan + commit"


def oracle_step(w, nthreads):
    from oracle import oracle_commit, oracle_tree_scan
    f = w.f64(0)
    oracle_tree_scan(f["x"], f["dt"], f["A"], f["B"], f["C"], f["D"], f["h0"], w.parent, nthreads=nthreads)
    oracle_commit(f["x"], f["dt"], f["A"], f["B"], f["h0"], w.parent, w.path, w.path_len, nthreads=nthreads)


def cpu_baseline(name, seconds):
    from oracle.walk import default_threads
    w, desc = oracle_sample(name)
    cores = default_threads()
    oracle_step(w, cores)                      # compile + warm
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_step(w, cores)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    nodes = w.batch * w.n_nodes * n
    return {"value": nodes / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{desc}; {n} repetitions in {el:.1f} s on {cores} threads (fp64 root-path walk)"}


def run_reference(args):
    from oracle.walk import default_threads
    w, desc = oracle_sample(args.config)
    cores = default_threads()
    K = args.steps or 3
    Wm = max(3, args.warmup)
    # Each step is one oracle pass over the bounded sample.
    for _ in range(min(Wm, 3)):
        oracle_step(w, cores)
    t0 = time.perf_counter()
    for _ in range(K):
        oracle_step(w, cores)
    el = time.perf_counter() - t0
    value = w.batch * w.n_nodes * K / el
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": K,
        "warmup": Wm, "ms_per_step": el * 1e3 / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {**workload_config(args.config, args.batch, args.layers), "sample": desc},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    out = run_ours(args, rank, world, local_rank)
    extras = [] if args.also in ("", "none") else [c for c in args.also.split(",") if c and c != args.config]
    if extras:
        import copy
        out["other_workloads"] = {}
        for name in extras:
            a2 = copy.copy(args)
            a2.config, a2.steps, a2.batch, a2.layers = name, None, None, None
            a2.no_e2e = args.no_e2e or name not in E2E_WORKLOADS
            o2 = run_ours(a2, rank, world, local_rank)
            r2 = o2["roofline"]
            out["other_workloads"][name] = {
                "value": o2["value"], "unit": o2["unit"], "ms_per_step": o2["ms_per_step"], "steps": o2["steps"],
                "sequences_per_s": o2["sequences_per_s"], "config": o2["config"], "clocks": o2["clocks"],
                "roofline": {k: r2[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "kernel",
                                                "bytes_per_launch", "kernel_ms_mean", "launch_ms_from",
                                                "kernel_ms_events", "frac_events")},
                "gpu_launches": o2["gpu_launches"],
            }
            for k in ("separate", "e2e"):
                if k in o2:
                    out["other_workloads"][name][k] = o2[k]
            if not args.no_unrolled and rank == 0 and name in SIDE_WORKLOADS:
                out["other_workloads"][name]["unrolled_baseline"] = unrolled_summary(o2, run_unrolled(name, local_rank))
            if not args.no_accept and rank == 0 and name in SIDE_WORKLOADS:
                out["other_workloads"][name]["accept_greedy"] = run_accept(name, args.vocab, local_rank)
                out["other_workloads"][name]["accept_sampling"] = run_sampling(name, args.vocab, local_rank)
            if not args.no_gdn and rank == 0 and name in SIDE_WORKLOADS:
                out["other_workloads"][name]["gdn_tree"] = run_gdn(name, local_rank)
                out["other_workloads"][name]["gla_tree"] = run_gdn(name, local_rank, linear=True)
            if not args.no_attention and rank == 0 and name in ATTN_CTX:
                out["other_workloads"][name]["tree_attention"] = run_attention(name, local_rank)
    if rank == 0 and not args.no_unrolled:
        out["unrolled_baseline"] = unrolled_summary(out, run_unrolled(args.config, local_rank))
    if rank == 0 and not args.no_accept:
        out["accept_greedy"] = run_accept(args.config, args.vocab, local_rank)
        out["accept_sampling"] = run_sampling(args.config, args.vocab, local_rank)
    if rank == 0 and not args.no_gdn:
        out["gdn_tree"] = run_gdn(args.config, local_rank)
        out["gla_tree"] = run_gdn(args.config, local_rank, linear=True)
    if rank == 0 and not args.no_attention and args.config in ATTN_CTX:
        out["tree_attention"] = run_attention(args.config, local_rank)
    if rank == 0 and not args.no_floor:
        out["latency_floor"] = run_floor(args.config, local_rank)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(args.config, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
