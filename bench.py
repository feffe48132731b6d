#!/usr/bin/env python
"""Throughput of the GRINQH batch-1 decode GEMV on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen3-8b-proj|uniform-sweep|70b|llama3-8b-step|gate-3b]
    python bench.py --workload prefill-qwen3-8b [--tokens T]

A step is one pass of the whole decode path over one token's inputs for every
linear of the workload: by default the fused grinqh_decode_gemv call per linear
(assignment, per-plane lists, counts and group sums written, then the GEMV, in
one kernel); with --path two, grinqh_assign then grinqh_gemv.  The
default workload is the Qwen3-8B-shaped projection set at batch 1 (q_proj
4096->4096, gate/up 4096->12288, down 12288->4096) at 2.0, 3.0 and 4.0
effective bits: 12 GEMVs per step, each with its own packed weights (504 MB of
planes, ~200 MB read per step, so consecutive steps do not hit in the 126 MB
L2).  Inputs are seeded synthetic: W ~ N(0, 0.02) quantized by 8-bit RTN,
x ~ N(0, 1) with 1% outliers x20, a fresh x per step from a pool of 8, and
static thresholds calibrated on 128 pooled draws.

The headline value is effective HBM bandwidth: the minimum bytes the method
must move (planes of the assigned widths, s/z of active groups, x, y) per
step, divided by the device time of the step.  One JSON line is printed by
rank 0.  With --gpus N > 1 (under torchrun) every rank runs its own replica of
the workload (weak scaling, no collective on the data path); the step time is
the max over ranks.

Beside the headline, the default line carries the per-GEMV cold-L2 table and
the dense 4-bit comparator (`cases`, `dense4`), the uniform-width sweep and its
linear fit (`latency_vs_bits`), a 70B-class pair (`seventy_b_class`), the
small-batch kernel at B = 2/4/8 (`small_batch`) and one prefill point
(`prefill`, 128 tokens, with cuBLAS on dense weights beside it).

--workload prefill-qwen3-8b times the other phase instead: a step is the
prefill GEMM (grinqh_prefill_gemm, every row at the full width b_max = 8) of
a block of T prompt tokens (default 128) through the same four Qwen3-8B
projections; the value is TFLOP/s (2 T d_in d_out per linear) against the
measured dense 16-bit tensor peak.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "µs per decode GEMV and effective HBM GB/s (fraction of B200 peak) vs eff. bits"
UNIT = "GB/s"
L2_BYTES = 126 * 1024 * 1024
N_POOL = 8
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (read + write) per launch of the dominant kernel on the
# qwen3-8b-proj step, from one ncu launch-list capture of this workload, keyed by
# the SHA-256 of the kernel source it was taken on: after any change to the
# kernel the figure no longer applies and the bench reports null.
NCU_TRAFFIC = {
    # gemv.cu, grinqh_gemv
    "84585736bc0dc9cf2ac9f0a4738586346a63ac0a4e44acbdc753bb3917df6db4": 17150844,
    # decode.cu, grinqh_decode_gemv (mean over the 60 launches of five steps)
    "c47d66cfdcd82c55fac824c3559139bcb3f01513339e270ed452c49dc315c372": 17345071,
}
KERNEL_SOURCE = {"fused": "decode.cu", "two": "gemv.cu"}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--path", choices=["fused", "two"], default="fused",
                    help="fused: grinqh_decode_gemv per linear; two: grinqh_assign + grinqh_gemv")
    ap.add_argument("--workload", default="qwen3-8b-proj",
                    choices=["qwen3-8b-proj", "uniform-sweep", "70b", "llama3-8b-step",
                             "gate-3b", "prefill-qwen3-8b"],
                    help="gate-3b: the single gate_proj 4096->12288 GEMV at 3 bits of the "
                         "qwen3-8b-proj set (a small case for profiler captures)")
    ap.add_argument("--tokens", type=int, default=128,
                    help="prefill-qwen3-8b: prompt tokens per step (T)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cases", action="store_true", help="skip the per-GEMV cold-L2 table")
    return ap.parse_args(argv)


def workload_specs(name):
    if name == "qwen3-8b-proj":
        return synth.config1()
    if name == "uniform-sweep":
        return synth.config2()
    if name == "70b":
        return synth.config3()
    if name == "llama3-8b-step":
        return synth.config4()
    if name == "gate-3b":
        return [s for s in synth.config1() if s.name == "gate_proj@3b"]
    raise ValueError(name)


def min_bytes(b: np.ndarray, d_out: int, include_x: bool = True) -> int:
    """Algorithmic bytes of one decode GEMV: the planes of the assigned widths,
    fp16 s and z of every group with an active row, x (fp16) and y (fp32)."""
    d_in = b.shape[0]
    planes = int(b.astype(np.int64).sum()) * d_out // 8
    g_act = int((b.reshape(-1, 128) > 0).any(axis=1).sum())
    return planes + 4 * d_out * g_act + (2 * d_in if include_x else 0) + 4 * d_out


def kernel_traffic(workload: str, path: str = "fused"):
    """ncu DRAM bytes per launch of the dominant kernel for its current source, or None."""
    if workload != "qwen3-8b-proj":
        return None
    import hashlib
    path = os.path.join(ROOT, "input_adaptive_bit_b200", "csrc", KERNEL_SOURCE[path])
    try:
        with open(path, "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    return NCU_TRAFFIC.get(digest)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            mp = json.load(f)
        return float(mp["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---- clocks during the timed region ---------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.t0 = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "20"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return []
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out = ""
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        return rows

    @staticmethod
    def summarize(rows):
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


# ---- the CUDA path ------------------------------------------------------------------

class Workload:
    """Device-resident layers, input pools and captured step graphs."""

    def __init__(self, specs, device, rank, path="fused"):
        import torch
        self.path = path
        from input_adaptive_bit_b200.layer import GrinqhLinear
        self.torch = torch
        self.device = device
        self.specs = specs
        self.layers, self.thetas = [], []
        cache = {}
        for spec in specs:
            # base codes are drawn once per distinct projection (name without the
            # bit-target / layer prefix); every linear still gets its own packed copy
            proj = (spec.d_in, spec.d_out, spec.b_max, spec.name.split("@")[0].split(".")[-1])
            if proj not in cache:
                g = synth.rng(spec.config_id, 1000 + len(cache), rank)
                W = synth.gaussian_weights(g, spec.d_in, spec.d_out)
                cache[proj] = synth.rtn_quantize(W, spec.b_max)
                del W
            q, s, z = cache[proj]
            self.layers.append(GrinqhLinear(q, s, z, spec.b_max, device=device))
            calib = synth.Linear(spec.name, spec.d_in, spec.d_out, spec.b_max, spec.target_bits,
                                 spec.uniform_b, spec.dist, spec.config_id, spec.layer,
                                 calib_draws=128 if spec.target_bits is not None else 0)
            x0 = synth.activations(synth.rng(spec.config_id, spec.layer, 0), spec.d_in, spec.dist)
            self.thetas.append(torch.from_numpy(synth.make_theta(calib, x0)).to(device))
        del cache
        # x pool: [N_POOL][sum d_in] fp16, host (pinned) and device copies
        self.offsets = np.cumsum([0] + [s.d_in for s in specs])
        self.y_offsets = np.cumsum([0] + [s.d_out for s in specs])
        xs = np.zeros((N_POOL, self.offsets[-1]), np.float16)
        for k in range(N_POOL):
            for j, spec in enumerate(specs):
                xs[k, self.offsets[j]:self.offsets[j + 1]] = synth.make_x(spec, 1000 * rank + k)
        self.x_host = torch.from_numpy(xs).pin_memory()
        self.x_dev = self.x_host.to(device)
        self.y_dev = torch.zeros(self.y_offsets[-1], dtype=torch.float32, device=device)
        self.y_host = torch.zeros(self.y_offsets[-1], dtype=torch.float32).pin_memory()
        self.stream = torch.cuda.Stream(device=device)
        self.graphs = []
        self.gemv_graph = None
        self.two_graph = None
        self.groups = self.layer_groups()
        self.group_graph = self.single_graph = None
        if self.groups is not None:
            from input_adaptive_bit_b200 import grinqh_group_workspace_bytes
            self.group_ws = torch.zeros(grinqh_group_workspace_bytes(), dtype=torch.uint8,
                                        device=device)

    def xv(self, k, j):
        return self.x_dev[k, self.offsets[j]:self.offsets[j + 1]]

    def yv(self, j):
        return self.y_dev[self.y_offsets[j]:self.y_offsets[j + 1]]

    def layer_groups(self):
        """The linears in launch order with the independent ones of a layer (q, k, v;
        gate, up) in one group each -- names "L<layer>.<kind>" or "<kind>_proj@<bits>";
        None when no two linears group."""
        groups, key_prev = [], None
        for j, spec in enumerate(self.specs):
            if "." in spec.name:
                layer, kind = spec.name.split(".", 1)
            elif "@" in spec.name:
                kind, layer = spec.name.split("@", 1)
            else:
                return None
            kind = kind.replace("_proj", "")
            key = (layer, {"q": "qkv", "k": "qkv", "v": "qkv", "gate": "gu", "up": "gu"}.get(kind, kind))
            if key == key_prev:
                groups[-1].append(j)
            else:
                groups.append([j])
            key_prev = key
        return None if all(len(g) == 1 for g in groups) else groups

    def launch_step_grouped(self, k, stream):
        """One step with each group of independent linears in one grouped launch (no
        optional outputs)."""
        from input_adaptive_bit_b200 import grinqh_decode_gemv_group
        for grp in self.groups:
            if len(grp) == 1:
                j = grp[0]
                self.layers[j].decode(self.xv(k, j), self.thetas[j], y=self.yv(j), outputs=False,
                                      stream=stream)
                continue
            lins = [(self.layers[j].planes, self.layers[j].s, self.layers[j].z, self.xv(k, j),
                     self.thetas[j], None, self.layers[j].d_in, self.layers[j].d_out,
                     self.layers[j].b_max, self.yv(j)) for j in grp]
            grinqh_decode_gemv_group(lins, self.group_ws, self.group_ws.numel(), stream=stream)

    def launch_step(self, k, stream, path=None, outputs=True):
        path = path or self.path
        for j, lin in enumerate(self.layers):
            if path == "fused":
                lin.decode(self.xv(k, j), self.thetas[j], y=self.yv(j), outputs=outputs,
                           stream=stream)
            else:
                lin.assign(self.xv(k, j), self.thetas[j], stream=stream)
                lin.gemv(self.yv(j), stream=stream)

    def launch_gemvs(self, stream):
        for j, lin in enumerate(self.layers):
            lin.gemv(self.yv(j), stream=stream)

    def capture(self):
        torch = self.torch
        with torch.cuda.stream(self.stream):
            for k in range(N_POOL):  # eager warm-up of every launch once, both paths
                self.launch_step(k, self.stream, "two")
                self.launch_step(k, self.stream, "fused")
        self.stream.synchronize()
        for k in range(N_POOL):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self.launch_step(k, self.stream)
            self.graphs.append(g)
        # the two-kernel path as a comparison: a whole step, and its gemv launches alone
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self.launch_step(0, self.stream, "two")
        self.two_graph = g
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self.launch_gemvs(self.stream)
        self.gemv_graph = g
        if self.groups is not None:  # layer stack: grouped launches, and the same without outputs
            with torch.cuda.stream(self.stream):
                self.launch_step_grouped(0, self.stream)
                self.launch_step(0, self.stream, outputs=False)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self.launch_step_grouped(0, self.stream)
            self.group_graph = g
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self.launch_step(0, self.stream, outputs=False)
            self.single_graph = g
        torch.cuda.synchronize(self.device)

    def bytes_per_pool_entry(self, include_x=True):
        """Algorithmic bytes of one step for each pool entry (needs b on the host)."""
        torch = self.torch
        out = []
        for k in range(N_POOL):
            self.graphs[k].replay()
            torch.cuda.synchronize(self.device)
            tot = 0
            for lin, spec in zip(self.layers, self.specs):
                tot += min_bytes(lin.b.cpu().numpy(), spec.d_out, include_x)
            out.append(tot)
        return out

    def effective_bits(self, k):
        torch = self.torch
        self.graphs[k].replay()
        torch.cuda.synchronize(self.device)
        return [float(lin.b.float().mean().item()) for lin in self.layers]


def device_time_ms(torch, stream, fn, n):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        fn(i)
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1)


class L2Flush:
    """Evicts the L2 by reading a 256 MB buffer (written once): the L2 is left
    holding clean lines, so the timed launch pays no write-back of a flush."""

    def __init__(self, torch, device):
        self.buf = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
        self.sink = torch.empty(1, dtype=torch.float32, device=device)

    def __call__(self):
        self.sink.copy_(self.buf.sum().reshape(1))


def _graph_ms(torch, st, body, reps):
    """Mean device ms of one replay of a graph that runs body() `reps` times."""
    with torch.cuda.stream(st):
        body()  # warm-up (first launches, smem attributes)
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            for _ in range(reps):
                body()
        g.replay()
        st.synchronize()
        ms = device_time_ms(torch, st, lambda i: g.replay(), 5)
    del g
    return ms / 5


def cold_case_times(wl, reps=20):
    """Per-GEMV device time with a cold L2: a graph of reps x (256 MB read, call)
    minus a graph of reps x (256 MB read), per call -- the fused decode call,
    assign + gemv, and gemv alone after an untimed assign."""
    torch = wl.torch
    flush = L2Flush(torch, wl.device)
    st = wl.stream
    t_flush = _graph_ms(torch, st, flush, reps) / reps
    rows = []
    for j, (lin, spec) in enumerate(zip(wl.layers[:16], wl.specs[:16])):
        xj, thj, yj = wl.xv(0, j), wl.thetas[j], wl.yv(j)

        def fused():
            flush()
            lin.decode(xj, thj, y=yj, stream=st)

        def two():
            flush()
            lin.assign(xj, thj, stream=st)
            lin.gemv(yj, stream=st)

        def assign_only():
            flush()
            lin.assign(xj, thj, stream=st)
            flush()

        def gemv_after_assign():
            flush()
            lin.assign(xj, thj, stream=st)
            flush()
            lin.gemv(yj, stream=st)

        med = {"fused": _graph_ms(torch, st, fused, reps) / reps - t_flush,
               "all": _graph_ms(torch, st, two, reps) / reps - t_flush,
               # both graphs hold the same two reads and assign: the difference is gemv
               "gemv": (_graph_ms(torch, st, gemv_after_assign, reps)
                        - _graph_ms(torch, st, assign_only, reps)) / reps}
        med = {k: v * 1e3 for k, v in med.items()}  # us
        b = lin.b.cpu().numpy()
        rows.append({"name": spec.name, "d_in": spec.d_in, "d_out": spec.d_out,
                     "b_max": spec.b_max, "eff_bits": round(float(b.mean()), 3),
                     "us_fused": round(med["fused"], 2),
                     "fused_GBps": round(min_bytes(b, spec.d_out) / (med["fused"] * 1e3), 1),
                     "us_assign_gemv": round(med["all"], 2),
                     "us_gemv": round(med["gemv"], 2),
                     "gemv_GBps": round(min_bytes(b, spec.d_out, False) / (med["gemv"] * 1e3), 1)})
    return rows


def dense4_times(wl, reps=20):
    """The in-library dense 4-bit comparator on each distinct shape, cold L2
    (graph of reps x (256 MB read, call) minus the reads)."""
    torch = wl.torch
    from input_adaptive_bit_b200.layer import Dense4Linear
    flush = L2Flush(torch, wl.device)
    st = wl.stream
    t_flush = _graph_ms(torch, st, flush, reps) / reps
    seen, rows = set(), []
    for j, spec in enumerate(wl.specs[:16]):
        if (spec.d_in, spec.d_out) in seen:
            continue
        seen.add((spec.d_in, spec.d_out))
        g = synth.rng(spec.config_id, 5000 + j, 0)
        q4, s, z = synth.rtn_quantize(synth.gaussian_weights(g, spec.d_in, spec.d_out), 4)
        d4 = Dense4Linear(q4, s, z, device=wl.device)
        xj = wl.xv(0, j)

        def call():
            flush()
            d4(xj, stream=st)

        t = (_graph_ms(torch, st, call, reps) / reps - t_flush) * 1e3
        nbytes = spec.d_in * spec.d_out // 2 + 4 * spec.d_out * (spec.d_in // 128) + 4 * spec.d_out
        rows.append({"name": f"dense4_{spec.d_in}x{spec.d_out}", "us": round(t, 2),
                     "GBps": round(nbytes / (t * 1e3), 1)})
        del d4
    return rows


def bits_fit(cases, specs):
    """Least-squares fit of fused latency against bits over the uniform-width
    cases (b_max 8): slope (us per bit), intercept and R^2."""
    pts = [(spec.uniform_b, c["us_fused"]) for c, spec in zip(cases, specs)
           if spec.uniform_b is not None and spec.b_max == 8]
    if len(pts) < 3:
        return None
    b = np.array([p[0] for p in pts], np.float64)
    t = np.array([p[1] for p in pts], np.float64)
    c, a = np.polyfit(b, t, 1)
    r2 = 1.0 - float(np.sum((t - (a + c * b)) ** 2)) / float(np.sum((t - t.mean()) ** 2))
    return {"us_per_bit": round(float(c), 3), "us_at_0_bits": round(float(a), 3),
            "r2": round(r2, 4), "points": [[int(x), round(float(y), 2)] for x, y in pts]}


def uniform_sweep_fit(device, reps=20):
    """Latency of the fused decode GEMV on the Llama-3-8B up_proj shape (4096 ->
    14336, b_max 8) with every row at the same width b in {2, 4, 6, 8}, cold L2,
    its least-squares fit against b, and the in-library dense 4-bit GEMV of the
    same shape (the same bytes as b = 4)."""
    import torch
    from input_adaptive_bit_b200.layer import Dense4Linear, GrinqhLinear
    spec = next(s for s in synth.config2() if s.b_max == 8)
    W = synth.gaussian_weights(synth.rng(spec.config_id, spec.layer, 0), spec.d_in, spec.d_out)
    q, s, z = synth.rtn_quantize(W, 8)
    lin = GrinqhLinear(q, s, z, 8, device=device)
    q4, s4, z4 = synth.rtn_quantize(W, 4)
    d4 = Dense4Linear(q4, s4, z4, device=device)
    del W, q, q4
    x = torch.from_numpy(synth.make_x(spec, 0)).to(device)
    y = torch.empty(spec.d_out, dtype=torch.float32, device=device)
    flush = L2Flush(torch, device)
    st = torch.cuda.Stream(device=device)
    t_flush = _graph_ms(torch, st, flush, reps) / reps
    pts = []
    for b in (2, 4, 6, 8):
        th = torch.from_numpy(synth.uniform_thresholds(b, 8)).to(device)

        def call(th=th):
            flush()
            lin.decode(x, th, y=y, outputs=False, stream=st)

        us = (_graph_ms(torch, st, call, reps) / reps - t_flush) * 1e3
        nbytes = min_bytes(np.full(spec.d_in, b, np.uint8), spec.d_out)
        pts.append((b, us, nbytes))

    def dense():
        flush()
        d4(x, y=y, stream=st)

    us_d4 = (_graph_ms(torch, st, dense, reps) / reps - t_flush) * 1e3
    # the same 4 bits per weight on the product's own machinery: a 4-bit base (b_max 4)
    # with every row read at full width is a dense 4-bit GEMV in the plane layout
    q4p, s4p, z4p = synth.rtn_quantize(
        synth.gaussian_weights(synth.rng(spec.config_id, spec.layer, 0), spec.d_in, spec.d_out), 4)
    lin4 = GrinqhLinear(q4p, s4p, z4p, 4, device=device)
    del q4p
    th4 = torch.from_numpy(synth.uniform_thresholds(4, 4)).to(device)

    def dense_same():
        flush()
        lin4.decode(x, th4, y=y, outputs=False, stream=st)

    us_d4s = (_graph_ms(torch, st, dense_same, reps) / reps - t_flush) * 1e3
    del lin4
    bits = np.array([p[0] for p in pts], np.float64)
    t = np.array([p[1] for p in pts], np.float64)
    c, a = np.polyfit(bits, t, 1)
    r2 = 1.0 - float(np.sum((t - (a + c * bits)) ** 2)) / float(np.sum((t - t.mean()) ** 2))
    d4_bytes = spec.d_in * spec.d_out // 2 + 4 * spec.d_out * (spec.d_in // 128) + 2 * spec.d_in \
        + 4 * spec.d_out
    return {"shape": "4096x14336 (b_max 8, every row at width b, cold L2)",
            "us_per_bit": round(float(c), 3), "us_at_0_bits": round(float(a), 3),
            "r2": round(r2, 4),
            "points": [{"bits": b, "us": round(u, 2), "GBps": round(n / (u * 1e3), 1)}
                       for b, u, n in pts],
            "dense4_us": round(us_d4, 2), "dense4_GBps": round(d4_bytes / (us_d4 * 1e3), 1),
            "time_4bit_vs_dense4": round(pts[1][1] / us_d4, 3),
            "dense4_same_kernel_us": round(us_d4s, 2),
            "dense4_same_kernel_GBps": round(d4_bytes / (us_d4s * 1e3), 1),
            "time_4bit_vs_dense4_same_kernel": round(pts[1][1] / us_d4s, 3),
            "dense4_how": "dense4: grinqh_gemv_dense4 (nibble layout, its own kernel); "
                          "dense4_same_kernel: grinqh_decode_gemv on a 4-bit base with every row "
                          "at width 4 (the same bytes, the product's kernel)"}


def seventy_b_pair(device, peak, n_pool=64, reps=4):
    """The 70B-class pair at 3 effective bits (8192 -> 28672 and 28672 -> 8192,
    Student-t x, Theta from 128 pooled calibration draws): fused decode GEMVs
    alternating between the two layers, a fresh x from a pool of n_pool per call
    (so the active rows change every call); 470 MB of planes, no flush."""
    import torch
    from input_adaptive_bit_b200.layer import GrinqhLinear
    specs = [s for s in synth.config3() if s.target_bits == 3.0]
    layers, thetas, pools = [], [], []
    for spec in specs:
        W = synth.gaussian_weights(synth.rng(spec.config_id, spec.layer, 0), spec.d_in, spec.d_out)
        q, s, z = synth.rtn_quantize(W, 8)
        del W
        layers.append(GrinqhLinear(q, s, z, 8, device=device))
        del q
        x0 = synth.activations(synth.rng(spec.config_id, spec.layer, 0), spec.d_in, spec.dist)
        thetas.append(torch.from_numpy(synth.make_theta(spec, x0)).to(device))
        pools.append(torch.from_numpy(np.stack([synth.make_x(spec, k) for k in range(n_pool)]))
                     .to(device))
    ys = [torch.empty(spec.d_out, dtype=torch.float32, device=device) for spec in specs]
    st = torch.cuda.Stream(device=device)
    # algorithmic bytes of every (layer, pool entry): widths from the kernel's own b output
    nbytes = [[0] * n_pool for _ in specs]
    eff = [[0.0] * n_pool for _ in specs]
    with torch.cuda.stream(st):
        for j, (lin, spec) in enumerate(zip(layers, specs)):
            for k in range(n_pool):
                lin.decode(pools[j][k], thetas[j], y=ys[j], stream=st)
                st.synchronize()
                b = lin.b.cpu().numpy()
                nbytes[j][k] = min_bytes(b, spec.d_out)
                eff[j][k] = float(b.mean())

    def body():
        for k in range(n_pool):
            for j, lin in enumerate(layers):
                lin.decode(pools[j][k], thetas[j], y=ys[j], outputs=False, stream=st)

    ms = _graph_ms(torch, st, body, 1)  # one replay = 2 n_pool GEMVs
    for _ in range(reps - 1):
        ms = min(ms, _graph_ms(torch, st, body, 1))
    total = sum(sum(v) for v in nbytes)
    us = ms * 1e3 / (2 * n_pool)
    gbps = total / (ms * 1e-3) / 1e9
    out = {"shapes": "8192x28672 and 28672x8192 alternating, 3 effective bits (target), "
                     "Student-t x, a fresh x per call from a pool of %d" % n_pool,
           "us_per_gemv": round(us, 2), "GBps": round(gbps, 1),
           "frac_of_hbm": round(gbps / peak, 4),
           "eff_bits": {spec.name: round(float(np.mean(e)), 3) for spec, e in zip(specs, eff)},
           "eff_bits_range": [round(min(min(e) for e in eff), 3), round(max(max(e) for e in eff), 3)]}
    del layers, pools
    torch.cuda.empty_cache()
    return out


def small_batch_sweep(device, reps=20, batches=(2, 4, 8)):
    """The small-batch decode step (grinqh_decode_gemv_batch) on the gate_proj shape
    (4096 -> 12288, b_max 8, Theta for 3 effective bits): B tokens, each its own
    seeded x, cold L2.  Bytes are the union's: planes of u_i = max_t b_t(i), s/z of
    groups with an active row, B inputs and B outputs."""
    import torch
    from input_adaptive_bit_b200 import grinqh_batch_workspace_bytes, grinqh_decode_gemv_batch
    from input_adaptive_bit_b200.layer import GrinqhLinear
    spec = next(s for s in synth.config1() if s.name == "gate_proj@3b")
    W = synth.gaussian_weights(synth.rng(spec.config_id, spec.layer, 0), spec.d_in, spec.d_out)
    q, s, z = synth.rtn_quantize(W, 8)
    del W
    lin = GrinqhLinear(q, s, z, 8, device=device)
    del q
    calib = synth.Linear(spec.name, spec.d_in, spec.d_out, 8, spec.target_bits, None, spec.dist,
                         spec.config_id, spec.layer, calib_draws=128)
    x0 = synth.activations(synth.rng(spec.config_id, spec.layer, 0), spec.d_in)
    theta = torch.from_numpy(synth.make_theta(calib, x0)).to(device)
    nws = grinqh_batch_workspace_bytes()
    ws = torch.zeros(nws, dtype=torch.uint8, device=device)
    flush = L2Flush(torch, device)
    st = torch.cuda.Stream(device=device)
    t_flush = _graph_ms(torch, st, flush, reps) / reps
    rows = []
    x1 = torch.from_numpy(synth.make_x(spec, 0)).to(device)
    y1 = torch.empty(spec.d_out, dtype=torch.float32, device=device)

    def one():
        flush()
        lin.decode(x1, theta, y=y1, outputs=False, stream=st)

    us1 = (_graph_ms(torch, st, one, reps) / reps - t_flush) * 1e3
    lin.decode(x1, theta, y=y1, stream=st)
    st.synchronize()
    b1 = lin.b.cpu().numpy()
    rows.append({"B": 1, "us": round(us1, 2), "union_eff_bits": round(float(b1.mean()), 3),
                 "GBps": round(min_bytes(b1, spec.d_out) / (us1 * 1e3), 1),
                 "kernel": "grinqh_decode_gemv"})
    for B in batches:
        X = torch.from_numpy(np.stack([synth.make_x(spec, k) for k in range(B)])).to(device)
        Y = torch.empty((B, spec.d_out), dtype=torch.float32, device=device)
        u = torch.empty(spec.d_in, dtype=torch.uint8, device=device)
        with torch.cuda.stream(st):
            grinqh_decode_gemv_batch(lin.planes, lin.s, lin.z, X, theta, None, B, spec.d_in,
                                     spec.d_out, 8, Y, u, ws, nws, stream=st)
        st.synchronize()
        un = u.cpu().numpy()

        def call(X=X, Y=Y, B=B):
            flush()
            grinqh_decode_gemv_batch(lin.planes, lin.s, lin.z, X, theta, None, B, spec.d_in,
                                     spec.d_out, 8, Y, None, ws, nws, stream=st)

        us = (_graph_ms(torch, st, call, reps) / reps - t_flush) * 1e3
        nbytes = min_bytes(un, spec.d_out) + (B - 1) * (2 * spec.d_in + 4 * spec.d_out)
        rows.append({"B": B, "us": round(us, 2), "union_eff_bits": round(float(un.mean()), 3),
                     "GBps": round(nbytes / (us * 1e3), 1),
                     "tokens_per_s": round(B / (us * 1e-6), 1),
                     "kernel": "grinqh_decode_gemv_batch"})
    return {"shape": "gate_proj 4096x12288 at 3 effective bits per token (b_max 8), cold L2",
            "points": rows}


# ---- the oracle on the host cores (baseline only) --------------------------------

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample_run(spec, rank=0, seconds=10.0, outs_per_rep=None, threads=None):
    """Times the oracle's assign + lists + gemv on one linear of the workload, on
    `threads` host threads (default: all).  Returns (GB/s-equivalent, threads,
    description)."""
    import oracle
    case = synth.make_case(spec)
    planes = oracle.pack(case.q, spec.b_max)  # offline step, not timed
    threads = threads or oracle.max_threads()
    n_out = spec.d_out if outs_per_rep is None else outs_per_rep
    outs = None if outs_per_rep is None else np.arange(n_out, dtype=np.int32)
    t0 = time.perf_counter()
    reps, moved = 0, 0
    while True:
        b = oracle.assign(case.x, case.theta, spec.b_max)
        oracle.lists(b, spec.b_max)
        oracle.gemv(planes, case.s, case.z, case.x, b, spec.b_max, outs=outs, threads=threads)
        reps += 1
        moved += min_bytes(b, spec.d_out) * n_out / spec.d_out
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    desc = (f"oracle assign+lists+gemv on {spec.name} ({spec.d_in}->{spec.d_out}), "
            f"{n_out} outputs per run, {reps} runs in {dt:.1f} s, "
            f"{'OpenMP over outputs' if threads > 1 else 'one thread'}")
    return moved / dt / 1e9, threads, desc


# ---- prefill workload ------------------------------------------------------------------

PREFILL_BMAX = 8
PREFILL_SETS = 2  # distinct weight sets, alternated step by step
PREFILL_SWEEP_T = (1, 16, 64, 128, 256, 512, 1024, 2048)


def prefill_point(device, T=128, steps=100):
    """The prefill GEMM of a T-token block through the four Qwen3-8B projections
    (the prefill workload's step), timed as in its own bench line, beside cuBLAS
    fp16 on dense weights of the same shapes; for the decode workload's line."""
    import torch
    wl = PrefillWorkload(T, device, 0)

    def run(graphs, i):
        graphs[i % PREFILL_SETS].replay()

    with torch.cuda.stream(wl.stream):
        for i in range(5):
            run(wl.graphs, i)
        ms = device_time_ms(torch, wl.stream, lambda i: run(wl.graphs, i), steps) / steps
    dgraphs, keep = wl.dense_graphs()
    with torch.cuda.stream(wl.stream):
        for i in range(3):
            run(dgraphs, i)
        ms_d = device_time_ms(torch, wl.stream, lambda i: run(dgraphs, i), steps) / steps
    flops = wl.flops
    del dgraphs, keep, wl
    torch.cuda.empty_cache()
    peak, kind = measured_tensor_peak(sustained=True)
    tf = flops / (ms * 1e-3) / 1e12
    return {"tokens": T, "shapes": "q 4096x4096, gate/up 4096x12288, down 12288x4096, b_max 8",
            "ms_per_step": round(ms, 5), "TFLOPs": round(tf, 1),
            "frac_of_tensor_peak": round(tf / peak, 4), "peak": peak, "peak_kind": kind,
            "cublas_fp16_dense_ms": round(ms_d, 5), "time_vs_cublas": round(ms / ms_d, 3),
            "kernel": "prefill_kernel (grinqh_prefill_gemm)"}


def measured_tensor_peak(sustained: bool):
    """Dense 16-bit tensor-core peak in TFLOP/s: the measured cuBLAS bf16 figure
    (fp16 has the same nominal dense rate on B200, ratio 1)."""
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)[key]), "measured " + key
    except Exception:
        return (1400.0 if sustained else 1590.0), "fallback"


def prefill_weights(g, d_in, d_out, b_max=PREFILL_BMAX):
    """Random base codes and fp16 s, z for a prefill layer; the prefill GEMM does
    the same work whatever the code values are."""
    q = g.integers(0, 1 << b_max, size=(d_in, d_out), dtype=np.uint8)
    s = (g.random((d_in // 128, d_out)) * 0.01 + 1e-4).astype(np.float16)
    z = (-(g.random((d_in // 128, d_out)) * 0.5)).astype(np.float16)
    return q, s, z


class PrefillWorkload:
    """PREFILL_SETS copies of the four Qwen3-8B projections (packed planes at
    b_max 8), a token block X per input width, fp32 outputs and one step graph
    per copy; plus fp16 dense weights of the same shapes for the cuBLAS
    comparator."""

    def __init__(self, T, device, rank):
        import torch
        from input_adaptive_bit_b200.layer import GrinqhLinear
        self.torch, self.device, self.T = torch, device, T
        self.shapes = list(synth.QWEN3_8B)
        self.sets = []
        for si in range(PREFILL_SETS):
            layers = []
            for li, (_, di, do) in enumerate(self.shapes):
                q, s, z = prefill_weights(synth.rng(5, 100 * si + li, rank), di, do)
                layers.append(GrinqhLinear(q, s, z, PREFILL_BMAX, device=device))
                del q
            self.sets.append(layers)
        widths = sorted({di for _, di, _ in self.shapes})
        g = synth.rng(5, 900, rank)
        self.x_host = {d: torch.from_numpy(synth.prefill_tokens(g, T, d)).pin_memory()
                       for d in widths}
        self.x_dev = {d: h.to(device) for d, h in self.x_host.items()}
        self.y_dev = [torch.zeros((T, do), dtype=torch.float32, device=device)
                      for _, _, do in self.shapes]
        self.y_host = [torch.zeros((T, do), dtype=torch.float32).pin_memory()
                       for _, _, do in self.shapes]
        self.stream = torch.cuda.Stream(device=device)
        self.flops = sum(2 * T * di * do for _, di, do in self.shapes)
        self.plane_bytes = sum(di * do * PREFILL_BMAX // 8 for _, di, do in self.shapes)
        self.graphs = [self._capture(lambda k=k: self.body(k)) for k in range(PREFILL_SETS)]

    def body(self, k):
        for lin, (_, di, _), y in zip(self.sets[k], self.shapes, self.y_dev):
            lin.prefill(self.x_dev[di], Y=y, stream=self.stream)

    def _capture(self, fn):
        torch, st = self.torch, self.stream
        with torch.cuda.stream(st):
            fn()  # first launches outside the capture (smem attributes)
            st.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                fn()
        return g

    def dense_graphs(self):
        """cuBLAS fp16 X @ W on the same shapes (PREFILL_SETS weight copies)."""
        torch = self.torch
        ws = [[torch.randn((di, do), dtype=torch.float16, device=self.device) * 0.02
               for _, di, do in self.shapes] for _ in range(PREFILL_SETS)]
        outs = [torch.empty((self.T, do), dtype=torch.float16, device=self.device)
                for _, _, do in self.shapes]

        def body(k):
            for w, (_, di, _), o in zip(ws[k], self.shapes, outs):
                torch.mm(self.x_dev[di], w, out=o)

        graphs = [self._capture(lambda k=k: body(k)) for k in range(PREFILL_SETS)]
        return graphs, (ws, outs)


def prefill_sweep(device, reps=10):
    """The gate_proj shape (4096 -> 12288) at several token counts, cold L2: a
    graph of reps x (256 MB read, call) minus a graph of reps x (256 MB read),
    for grinqh_prefill_gemm and for cuBLAS fp16 on dense weights."""
    import torch
    from input_adaptive_bit_b200.layer import GrinqhLinear
    di, do = 4096, 12288
    q, s, z = prefill_weights(synth.rng(5, 950, 0), di, do)
    lin = GrinqhLinear(q, s, z, PREFILL_BMAX, device=device)
    del q
    w16 = torch.randn((di, do), dtype=torch.float16, device=device) * 0.02
    flush = L2Flush(torch, device)
    st = torch.cuda.Stream(device=device)
    t_flush = _graph_ms(torch, st, flush, reps) / reps
    g = synth.rng(5, 951, 0)
    rows = []
    for T in PREFILL_SWEEP_T:
        X = torch.from_numpy(synth.prefill_tokens(g, T, di)).to(device)
        Y = torch.empty((T, do), dtype=torch.float32, device=device)
        Yh = torch.empty((T, do), dtype=torch.float16, device=device)

        def ours():
            flush()
            lin.prefill(X, Y=Y, stream=st)

        def dense():
            flush()
            torch.mm(X, w16, out=Yh)

        us = (_graph_ms(torch, st, ours, reps) / reps - t_flush) * 1e3
        us_d = (_graph_ms(torch, st, dense, reps) / reps - t_flush) * 1e3
        fl = 2.0 * T * di * do
        rows.append({"T": T, "us": round(us, 2), "TFLOPs": round(fl / (us * 1e-6) / 1e12, 1),
                     "plane_GBps": round(di * do / (us * 1e3), 1),
                     "cublas_fp16_us": round(us_d, 2),
                     "cublas_fp16_TFLOPs": round(fl / (us_d * 1e-6) / 1e12, 1),
                     "time_vs_cublas": round(us / us_d, 3)})
    return rows


def oracle_prefill_sample(seconds=10.0, threads=None):
    """The oracle's full-width GEMV of one token after another on q_proj
    (4096 -> 4096).  Returns (TFLOP/s, threads, description)."""
    import oracle
    di, do = 4096, 4096
    q, s, z = prefill_weights(synth.rng(5, 960, 0), di, do)
    planes = oracle.pack(q, PREFILL_BMAX)  # offline step, not timed
    X = synth.prefill_tokens(synth.rng(5, 961, 0), 64, di)
    full = np.full(di, PREFILL_BMAX, np.uint8)
    threads = threads or oracle.max_threads()
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.gemv(planes, s, z, X[n % len(X)], full, PREFILL_BMAX, threads=threads)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    desc = (f"oracle full-width gemv of {n} tokens on q_proj (4096->4096) in {dt:.1f} s, "
            f"{'OpenMP over outputs' if threads > 1 else 'one thread'}")
    return 2.0 * di * do * n / dt / 1e12, threads, desc


def run_prefill(args):
    import torch
    rank, world, dist = init_dist(torch)
    device = torch.device("cuda", torch.cuda.current_device())
    from input_adaptive_bit_b200 import lib
    lib()  # fail loudly if the CUDA library is missing
    T = args.tokens
    wl = PrefillWorkload(T, device, rank)
    props = torch.cuda.get_device_properties(device)
    try:
        gpu_id = "GPU-" + str(props.uuid)
    except Exception:
        gpu_id = None
    sampler = ClockSampler(gpu_id)

    def barrier():
        torch.cuda.synchronize(device)
        if dist is not None:
            dist.barrier()

    def run(graphs, i):
        graphs[i % PREFILL_SETS].replay()

    with torch.cuda.stream(wl.stream):
        for i in range(args.warmup):
            run(wl.graphs, i)
    barrier()
    sampler.start()
    time.sleep(0.3)
    barrier()
    with torch.cuda.stream(wl.stream):
        ms = device_time_ms(torch, wl.stream, lambda i: run(wl.graphs, i), args.steps)
    barrier()
    time.sleep(0.1)
    clocks = ClockSampler.summarize(sampler.stop())
    ms = max_over_ranks(dist, ms, device)
    ms_step = ms / args.steps
    value = world * wl.flops * args.steps / (ms * 1e-3) / 1e12

    # cuBLAS fp16 on dense weights of the same shapes, same protocol
    dgraphs, keep = wl.dense_graphs()
    reps = max(20, min(1000, args.steps))
    with torch.cuda.stream(wl.stream):
        for i in range(3):
            run(dgraphs, i)
        ms_d = device_time_ms(torch, wl.stream, lambda i: run(dgraphs, i), reps)
    ms_d = max_over_ranks(dist, ms_d, device) / reps
    del dgraphs, keep

    # end to end: pinned X H2D, the step, Y D2H, host sync, every step
    k_e2e = max(10, min(args.steps, 200))
    h2d = sum(h.numel() * 2 for h in wl.x_host.values())
    d2h = sum(h.numel() * 4 for h in wl.y_host)

    def e2e_step(i):
        for d, h in wl.x_host.items():
            wl.x_dev[d].copy_(h, non_blocking=True)
        run(wl.graphs, i)
        for yd, yh in zip(wl.y_dev, wl.y_host):
            yh.copy_(yd, non_blocking=True)
        wl.stream.synchronize()

    barrier()
    with torch.cuda.stream(wl.stream):
        for i in range(3):
            e2e_step(i)
        t0 = time.perf_counter()
        ms_e2e = device_time_ms(torch, wl.stream, e2e_step, k_e2e)
        wall = (time.perf_counter() - t0) * 1e3
    ms_e2e = max_over_ranks(dist, max(ms_e2e, wall), device)
    e2e_value = world * wl.flops * k_e2e / (ms_e2e * 1e-3) / 1e12

    sweep = None
    if rank == 0 and not args.no_cases:
        sweep = prefill_sweep(device)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, threads, desc = oracle_prefill_sample(10.0)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": desc, "cpu_model": cpu_model()}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peak, peak_kind = measured_tensor_peak(sustained=True)
    burst, _ = measured_tensor_peak(sustained=False)
    hbm, hbm_kind = measured_peaks()
    achieved = wl.flops / (ms_step * 1e-3) / 1e12
    line = {
        "metric": "prefill GEMM TFLOP/s at full width b_max 8", "value": round(value, 1),
        "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 x f16 -> f32", "data": "synthetic",
        "config": {"workload": "prefill of a %d-token block through the qwen3-8b projections "
                               "(q 4096x4096, gate/up 4096x12288, down 12288x4096), every row "
                               "at b_max 8" % T,
                   "tokens": T, "gemms_per_step": len(wl.shapes),
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: steps alternate between %d copies of the "
                         "weights, %d MB of planes in all; no flush" % (
                             PREFILL_SETS, PREFILL_SETS * wl.plane_bytes // 2**20),
                   "flops_per_step": wl.flops, "plane_bytes_per_step": wl.plane_bytes},
        "roofline": {"bound": "tensor", "kernel": "prefill_kernel (grinqh_prefill_gemm)",
                     "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "frac_of_burst": round(achieved / burst, 4), "traffic": None,
                     "hbm_view": {"plane_GBps": round(wl.plane_bytes / (ms_step * 1e-3) / 1e9, 1),
                                  "peak": hbm, "peak_kind": hbm_kind},
                     "how": "2 T d_in d_out per linear over the step's device time; the "
                            "step also holds each call's memset of Y"},
        "cublas_fp16_dense": {"ms_per_step": round(ms_d, 5),
                              "TFLOPs": round(wl.flops / (ms_d * 1e-3) / 1e12, 1),
                              "time_ratio": round(ms_step / ms_d, 3),
                              "how": "torch.mm on fp16 weights of the same shapes, "
                                     "%d weight copies alternated" % PREFILL_SETS},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": k_e2e,
                "how": "pinned X H2D + step graph + Y D2H + host sync, every step"},
        "gpu_launches": len(wl.shapes) * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if sweep is not None:
        line["sweep_gate_4096x12288"] = sweep
    print(json.dumps(line), flush=True)
    return 0


# ---- main ------------------------------------------------------------------------------

def max_over_ranks(dist, v: float, device) -> float:
    """The largest v over all ranks (v itself without a process group)."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbps(world: int, bytes_per_rank: float, ms: float) -> float:
    """Weak scaling: every rank moved bytes_per_rank in at most ms (the max over ranks)."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(torch):
    """(rank, world, torch.distributed or None); one process per GPU over NCCL."""
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return rank, world, dist
    torch.cuda.set_device(0)
    return rank, world, None


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    # the whole run stays near two minutes whatever K and W are; every step does
    # at least one full sample
    budget = min(20.0, 120.0 / max(1, args.steps + args.warmup))
    if args.workload == "prefill-qwen3-8b":
        metric, unit, dtype = "prefill GEMM TFLOP/s at full width b_max 8", "TFLOP/s", "f64"
        sample = lambda sec: oracle_prefill_sample(sec)  # noqa: E731
        sampled = "q_proj 4096->4096"
    else:
        metric, unit, dtype = METRIC, UNIT, "f64"
        spec = min(workload_specs(args.workload), key=lambda s: s.d_in * s.d_out)
        sample = lambda sec: oracle_sample_run(spec, seconds=sec, outs_per_rep=512)  # noqa: E731
        sampled = spec.name
    vals = []
    for _ in range(args.warmup):
        sample(budget / 4)
    t0 = time.perf_counter()
    threads, desc = 0, ""
    for _ in range(args.steps):
        v, threads, desc = sample(budget)
        vals.append(v)
    dt = time.perf_counter() - t0
    value = float(np.mean(vals)) if vals else 0.0
    line = {"impl": "reference", "metric": metric, "value": round(value, 6), "unit": unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * dt / max(1, args.steps), 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
            "config": {"workload": args.workload, "sampled_linear": sampled},
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)

    if args.workload == "prefill-qwen3-8b":
        return run_prefill(args)
    import torch
    rank, world, dist = init_dist(torch)
    device = torch.device("cuda", torch.cuda.current_device())

    from input_adaptive_bit_b200 import lib
    lib()  # fail loudly if the CUDA library is missing

    specs = workload_specs(args.workload)
    wl = Workload(specs, device, rank, args.path)
    wl.capture()
    step_bytes = wl.bytes_per_pool_entry(include_x=True)
    gemv_bytes = wl.bytes_per_pool_entry(include_x=False)
    eff_bits = wl.effective_bits(0)

    props = torch.cuda.get_device_properties(device)
    gpu_id = None
    try:
        gpu_id = "GPU-" + str(props.uuid)
    except Exception:
        gpu_id = None
    sampler = ClockSampler(gpu_id)

    def barrier():
        torch.cuda.synchronize(device)
        if dist is not None:
            dist.barrier()


    # warm-up
    with torch.cuda.stream(wl.stream):
        for i in range(args.warmup):
            wl.graphs[i % N_POOL].replay()
    barrier()

    # ---- timed region: K steps --------------------------------------------------
    sampler.start()
    time.sleep(0.3)
    barrier()
    with torch.cuda.stream(wl.stream):
        ms = device_time_ms(torch, wl.stream, lambda i: wl.graphs[i % N_POOL].replay(), args.steps)
    barrier()
    time.sleep(0.1)
    clocks = ClockSampler.summarize(sampler.stop())
    ms = max_over_ranks(dist, ms, device)
    bytes_timed = sum(step_bytes[i % N_POOL] for i in range(args.steps))
    value = whole_job_gbps(world, bytes_timed, ms)
    n_gemv = len(specs)

    # ---- the dominant kernel -------------------------------------------------------
    # fused: the step is n_gemv launches of the one decode kernel, timed above;
    # two: grinqh_gemv alone over the same layers (after an assign of pool entry 0)
    reps = max(20, min(2000, args.steps))
    with torch.cuda.stream(wl.stream):
        wl.two_graph.replay()
        ms_g = device_time_ms(torch, wl.stream, lambda i: wl.gemv_graph.replay(), reps)
        ms_two = device_time_ms(torch, wl.stream, lambda i: wl.two_graph.replay(), reps)
    ms_g = max_over_ranks(dist, ms_g, device)
    ms_two = max_over_ranks(dist, ms_two, device)
    gemv_launch_us = ms_g * 1e3 / (reps * n_gemv)
    peak, peak_kind = measured_peaks()
    if args.path == "fused":
        kernel_name = "decode_kernel (grinqh_decode_gemv)"
        launch_us = ms * 1e3 / (args.steps * n_gemv)
        bytes_launch = bytes_timed / (args.steps * n_gemv)
    else:
        kernel_name = "gemv_kernel (grinqh_gemv)"
        launch_us = gemv_launch_us
        bytes_launch = gemv_bytes[0] / n_gemv
    achieved = bytes_launch / (launch_us * 1e-6) / 1e9
    grouped = None
    if wl.group_graph is not None:
        with torch.cuda.stream(wl.stream):
            ms_grp = device_time_ms(torch, wl.stream, lambda i: wl.group_graph.replay(), reps)
            ms_one = device_time_ms(torch, wl.stream, lambda i: wl.single_graph.replay(), reps)
        ms_grp = max_over_ranks(dist, ms_grp, device)
        ms_one = max_over_ranks(dist, ms_one, device)
        grouped = {"launches_per_step": len(wl.groups),
                   "ms_per_step": round(ms_grp / reps, 5),
                   "value": round(step_bytes[0] / (ms_grp / reps * 1e-3) / 1e9, 1),
                   "ungrouped_no_outputs_ms_per_step": round(ms_one / reps, 5),
                   "how": "the independent linears of a layer (q/k/v, gate/up) in one "
                          "grinqh_decode_gemv_group launch; no optional outputs in either graph; "
                          "pool entry 0"}
    two_kernel = {"ms_per_step": round(ms_two / reps, 5),
                  "value": round(step_bytes[0] / (ms_two / reps * 1e-3) / 1e9, 1),
                  "gemv_us_per_launch": round(gemv_launch_us, 3),
                  "gemv_GBps": round(gemv_bytes[0] / n_gemv / (gemv_launch_us * 1e-6) / 1e9, 1)}

    # ---- end to end through the public API with host buffers --------------------
    k_e2e = max(10, min(args.steps, 500))
    xbytes = wl.x_host[0].numel() * 2
    ybytes = wl.y_host.numel() * 4

    def e2e_step(i):
        k = i % N_POOL
        wl.x_dev[k].copy_(wl.x_host[k], non_blocking=True)
        wl.graphs[k].replay()
        wl.y_host.copy_(wl.y_dev, non_blocking=True)
        wl.stream.synchronize()

    barrier()
    with torch.cuda.stream(wl.stream):
        for i in range(3):
            e2e_step(i)
        t0 = time.perf_counter()
        ms_e2e = device_time_ms(torch, wl.stream, e2e_step, k_e2e)
        wall_e2e = (time.perf_counter() - t0) * 1e3
    ms_e2e = max_over_ranks(dist, max(ms_e2e, wall_e2e), device)
    e2e_bytes = sum(step_bytes[i % N_POOL] for i in range(k_e2e))
    e2e_value = whole_job_gbps(world, e2e_bytes, ms_e2e)

    planes_mb = sum(lin.planes.numel() * 4 for lin in wl.layers) // 2**20
    cases = None
    dense4 = None
    sweep_fit = seventy = small_batch = prefill = None
    if not args.no_cases and rank == 0:
        cases = cold_case_times(wl)
        dense4 = dense4_times(wl)
        if args.workload == "qwen3-8b-proj":
            peak_hbm, _ = measured_peaks()
            del wl
            torch.cuda.empty_cache()
            sweep_fit = uniform_sweep_fit(device)
            seventy = seventy_b_pair(device, peak_hbm)
            small_batch = small_batch_sweep(device)
            prefill = prefill_point(device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        spec = next(s for s in specs if s.d_in * s.d_out == min(x.d_in * x.d_out for x in specs))
        v, threads, desc = oracle_sample_run(spec, seconds=10.0)
        v1, _, desc1 = oracle_sample_run(spec, seconds=5.0, threads=1)
        cpu = {"value": round(v, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc, "cpu_model": cpu_model(),
               "single_thread": {"value": round(v1, 4), "sample": desc1}}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": args.workload if args.workload != "qwen3-8b-proj"
                   else "qwen3-8b projections at batch 1 (q 4096x4096, gate/up 4096x12288, "
                        "down 12288x4096) x {2.0, 3.0, 4.0} effective bits, b_max 8",
                   "gemvs_per_step": n_gemv, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: each step reads ~%d MB of planes from %d MB of "
                         "distinct packed weights; no flush" % (
                             gemv_bytes[0] // 2**20,
                             planes_mb),
                   "eff_bits": [round(e, 3) for e in eff_bits],
                   "us_per_gemv": round(ms * 1e3 / (args.steps * n_gemv), 3),
                   "bytes_per_step": int(np.mean(step_bytes))},
        "roofline": {"bound": "hbm", "kernel": kernel_name, "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": kernel_traffic(args.workload, args.path),
                     "bytes_per_launch": int(bytes_launch),
                     "us_per_launch": round(launch_us, 3)},
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": int(xbytes),
                "d2h_bytes_per_step": int(ybytes), "steps": k_e2e,
                "how": "pinned x H2D + step graph of the library calls + y D2H + host sync, "
                       "every step"},
        "gpu_launches": (1 if args.path == "fused" else 2) * n_gemv * args.steps,
        "path": args.path,
        "two_kernel_path": two_kernel,
        **({"grouped_layers": grouped} if grouped is not None else {}),
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if cases is not None:
        line["cases"] = cases
        line["dense4"] = dense4
        fit = bits_fit(cases, specs)
        if fit is not None:
            line["latency_vs_bits"] = fit
    if sweep_fit is not None:
        line["latency_vs_bits"] = sweep_fit
    if seventy is not None:
        line["seventy_b_class"] = seventy
    if small_batch is not None:
        line["small_batch"] = small_batch
    if prefill is not None:
        line["prefill"] = prefill
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
