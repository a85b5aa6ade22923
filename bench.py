#!/usr/bin/env python
"""Throughput of the fused DiT token operators on B200.

    python bench.py [--gpus N [--split]] [--steps K] [--warmup W] [--impl dit|reference]
                    [--workload batched_varlen] [--seed 0]
                    [--table | --variants | --host-overhead | --launch-cost]

One step runs the whole per-token hot path once over one packed batch:
Q/K RMSNorm + RoPE (in place), adaLN modulation, gated residual and SwiGLU,
each on its own synthetic buffers of the workload's shapes.  The default
workload is the largest single-GPU one, "batched_varlen": 4 requests with
seeded lengths in [1024, 30000] (69,829 valid tokens at seed 0), hidden 5120,
40 heads x 128, SwiGLU inner 13824, 3D RoPE on 24x42 latent frames plus a 1D
tail.  Every op's working set (>= 1.4 GB) is larger than the 126 MB L2, so no
flush is needed between steps.

Timing: W untimed steps, then exactly K steps on the launch stream with a
CUDA event at every step boundary (median, p10 and p90 per step in
``step_spread``), a barrier + synchronize on both sides, the max over ranks.
Rank 0 prints one JSON line.  ``value`` is tokens/s over all ranks; ``e2e``
repeats the measurement through the same public API with the inputs copied
from pinned host memory and the outputs copied back inside the timed region;
``roofline`` rates the dominant kernel against the measured HBM copy
bandwidth; ``clocks`` summarises NVML samples (every 5 ms) of the timed
window; ``small_shapes`` times the step at the per-rank-sized shapes
(single_stream, and long_video_slice: one rank's share of the long video
under an 8-way row split) against the sum of the ops timed alone;
``cpu_baseline`` times the plain CPU oracle on a bounded sample, on all host
threads and on one.

``--gpus N`` (under torch.distributed.run) gives every rank its own batch
(weak scaling); with ``--split`` the ranks instead split ONE batch by valid
tokens (``dit_token_b200.shard``, strong scaling), with no exchange.

``--impl reference`` times the CPU oracle alone (the only reference this
operator set has): rank 0 runs K + W bounded samples of the same workload on
the host cores and prints the same JSON line with "impl": "reference".

``--table`` prints a per-op markdown table over every workload and
``--variants`` one over the operator variants (fp32 and per-stream
modulation vectors, rotary layouts, grouped K heads, head_dim 256), both
with a read-only pass over 512 MB before every timed launch (clean L2);
``--host-overhead`` prints the host time per call of every entry point, and
``--launch-cost`` the device time of one call alone and per call in a chain
of calls on separate buffer sets at the small shapes.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from dit_token_b200 import workloads as W  # noqa: E402

METRIC = "fused DiT token-op throughput (tokens/s, achieved HBM GB/s, % of roofline) on 1 B200"
UNIT = "tokens/s"
OPS = ("qk_rmsnorm_rope", "adaln_modulate", "gated_residual", "swiglu")
FALLBACK_HBM_GBS = 6650.0
FRAMES_ELEMS = 1 * 3 * 243 * 768 * 1344
PROFILES = os.path.join(ROOT, "profiles")


# ------------------------------------------------------------ accounting

def algorithmic_bytes(w: W.Workload) -> dict:
    """HBM bytes each op must move per step: valid rows only, bf16.
    qk: q and k read + written (4 bytes per element of each); adaLN: x read,
    out written (4 C); gated residual: x, y read, out written (6 C); SwiGLU:
    a, b read, out written (6 I).  Per-sequence vectors, norm weights and the
    packing descriptors are O(num_seqs * C) and left out."""
    n = w.num_valid
    qk_elems = (w.num_q_heads + w.num_k_heads) * w.head_dim
    return {"qk_rmsnorm_rope": 4 * qk_elems * n, "adaln_modulate": 4 * w.hidden * n,
            "gated_residual": 6 * w.hidden * n, "swiglu": 6 * w.inner * n}


def _code_only(text: str) -> str:
    """C/C++ source with comments removed and whitespace collapsed: the digest
    follows the code, not its commentary."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_digest(op: str) -> str:
    """Digest of the code of an op's kernel file and of the shared device
    header (comments and layout ignored)."""
    csrc = os.path.join(ROOT, "dit_token_b200", "csrc")
    h = hashlib.sha256()
    for name in (f"{op}.cu", "common.cuh"):
        with open(os.path.join(csrc, name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(op: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, or None when there is none or the kernel changed since."""
    path = os.path.join(PROFILES, f"{op}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    d = re.search(r"kernel_source_digest:\s*([0-9a-f]+)", text)
    if not m or not d or d.group(1) != kernel_source_digest(op):
        return None
    return float(m.group(1))


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU while the work runs.

    Polls NVML every 5 ms from a background thread (query only: nothing is
    set), so even a timed region of a few tens of milliseconds holds several
    samples; falls back to ``nvidia-smi -lms 200`` where NVML is unavailable."""
    # NVML clock-event reason bits that the summary names
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int, period_s: float = 0.005):
        self.samples = []   # (host time, sm MHz, reason names, power W)
        self.period = period_s
        self.proc = None
        self.stop_flag = threading.Event()
        self.thread = None
        self.source = None
        self.max_mhz = None
        try:
            ident = str(torch.cuda.get_device_properties(device).uuid)
            ident = ident if ident.startswith("GPU-") else "GPU-" + ident
        except Exception:
            ident = str(device)
        self.ident = ident

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.ident.encode() if isinstance(self.ident, str) else self.ident)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.source = f"nvml every {self.period * 1e3:.0f} ms"

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        t = time.time()
                        sm = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        bits = int(get_reasons(h))
                        pw = pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                        names = [n for n, b in self.REASON_BITS.items() if bits & b]
                        self.samples.append((t, sm, names, pw))
                    except Exception:
                        return
                    self.stop_flag.wait(self.period)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.source = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 f"--id={self.ident}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi every 200 ms"
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None

    def _read(self):
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 9:
                continue
            try:
                sm = float(parts[1])
                self.max_mhz = float(parts[2])
                pw = float(parts[3])
            except ValueError:
                continue
            active = [n for n, v in zip(names, parts[5:9]) if v.lower() == "active"]
            self.samples.append((time.time(), sm, active, pw))

    def stop(self):
        self.stop_flag.set()
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        """Median, min and max SM clock, reasons seen and peak power over the
        samples taken inside [t0, t1] (all samples if none fell inside)."""
        window = [p for p in self.samples if t0 <= p[0] <= t1]
        rows = window or self.samples
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": self.source}
        sm = [r[1] for r in rows]
        reasons = sorted({n for r in rows for n in r[2]})
        return {"sm_mhz": statistics.median(sm), "sm_mhz_min": min(sm), "sm_mhz_max": max(sm),
                "sm_max_mhz": self.max_mhz, "power_w_max": round(max(r[3] for r in rows), 1),
                "reasons": reasons, "samples": len(rows), "in_timed_window": bool(window),
                "window_s": round(t1 - t0, 4), "source": self.source}


def clock_note(sampler: ClockSampler) -> str:
    """One line on the SM clock over a whole --table / --variants run."""
    sampler.stop()
    c = sampler.summary(float("-inf"), float("inf"))
    if not c["samples"]:
        return "\nSM clock: not sampled (no NVML or nvidia-smi)"
    return (f"\nSM clock over the run: median {c['sm_mhz']:.0f} MHz (min {c['sm_mhz_min']:.0f}, max "
            f"{c['sm_mhz_max']:.0f}; clocks.max.sm {c['sm_max_mhz']:.0f}), reasons {c['reasons'] or 'none'}, "
            f"peak power {c['power_w_max']} W, {c['samples']} samples ({c['source']})")


def spread(values_ms) -> dict:
    """Median, 10th and 90th percentile of per-step (or per-launch) times, in us."""
    v = np.asarray(list(values_ms), dtype=np.float64) * 1e3
    return {"median_us": round(float(np.median(v)), 2), "p10_us": round(float(np.percentile(v, 10)), 2),
            "p90_us": round(float(np.percentile(v, 90)), 2), "n": int(v.size)}


# ------------------------------------------------------------ distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def data_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch (same lengths, different values)."""
    return seed + 1000003 * rank


def reduce_max(value: float, device) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------ GPU arm

class Step:
    """Device buffers of one step and the four calls through the binding."""

    def __init__(self, w: W.Workload, host: dict, device):
        import dit_token_b200 as dit
        self.dit = dit
        self.w = w
        dev = lambda t: t.to(device, non_blocking=False)
        self.cs = torch.from_numpy(w.cu_seqlens).to(device)
        self.cp = torch.from_numpy(w.cu_seqlens_padded).to(device)
        self.grid = None if w.rope_grid is None else torch.from_numpy(w.rope_grid).to(device)
        self.pos_offset = None if w.pos_offset is None else torch.from_numpy(w.pos_offsets).to(device)
        self.q, self.k = dev(host["qk"]["q"]), dev(host["qk"]["k"])
        self.wq, self.wk = dev(host["qk"]["q_weight"]), dev(host["qk"]["k_weight"])
        self.ax, self.aout = dev(host["adaln"]["x"]), dev(host["adaln"]["out"])
        self.mod = dev(host["adaln"]["mod"])
        self.rx, self.ry, self.rout = dev(host["res"]["x"]), dev(host["res"]["y"]), dev(host["res"]["out"])
        self.ab, self.sout = dev(host["swiglu"]["ab"]), dev(host["swiglu"]["out"])
        # the views each call takes, made once (as a caller holding its
        # activations would), so the per-call host work is the binding's own
        rv = W.rows_view
        self.v = {"q": rv(self.q), "k": rv(self.k), "ax": rv(self.ax), "aout": rv(self.aout),
                  "rx": rv(self.rx), "ry": rv(self.ry), "rout": rv(self.rout), "sout": rv(self.sout),
                  "a": rv(self.ab)[:, : w.inner], "b": rv(self.ab)[:, w.inner:],
                  "shift": self.mod[:, 0], "scale": self.mod[:, 1], "gate": self.mod[:, 2]}

    def op_inputs(self, op):
        """Device tensors an op reads (what a host-resident caller must upload)."""
        return {"qk_rmsnorm_rope": [self.q, self.k], "adaln_modulate": [self.ax],
                "gated_residual": [self.rx, self.ry], "swiglu": [self.ab]}[op]

    def op_outputs(self, op):
        """Device tensors an op writes (what the caller reads back)."""
        return {"qk_rmsnorm_rope": [self.q, self.k], "adaln_modulate": [self.aout],
                "gated_residual": [self.rout], "swiglu": [self.sout]}[op]

    def run_op(self, op):
        w, d, v = self.w, self.dit, self.v
        if op == "qk_rmsnorm_rope":
            d.dit_qk_rmsnorm_rope(v["q"], v["k"], self.wq, self.wk, self.cs, self.cp,
                                  num_q_heads=w.num_q_heads, num_k_heads=w.num_k_heads, head_dim=w.head_dim,
                                  rope_grid=self.grid, sections=w.sections, rope_theta=w.rope_theta, eps=w.eps,
                                  pos_offset=self.pos_offset)
        elif op == "adaln_modulate":
            d.dit_adaln_modulate(v["ax"], v["shift"], v["scale"], self.cs, self.cp, out=v["aout"], eps=w.eps)
        elif op == "gated_residual":
            d.dit_gated_residual(v["rx"], v["ry"], v["gate"], self.cs, self.cp, out=v["rout"])
        else:
            d.dit_swiglu(v["a"], v["b"], self.cs, self.cp, out=v["sout"])

    def run(self, events=None):
        for op in OPS:
            if events:
                events[op][0].record()
            self.run_op(op)
            if events:
                events[op][1].record()


def frames_shape(scale: float = 1.0):
    """Decoded-frame tensor of the pages' request, its frame count scaled with
    the workload."""
    B, C, T, H, Wd = W.FRAMES_SHAPE
    return (B, C, max(1, int(round(T * scale))), H, Wd)


def time_next_ops(step: Step, steps: int, warmup: int, device, scale: float = 1.0) -> dict:
    """Mean launch time of the operators built beyond the four-op step (same
    buffers, same stream), each timed on its own."""
    w, d, rv = step.w, step.dit, W.rows_view

    def fused():
        d.dit_gated_residual_adaln(rv(step.rx), rv(step.ry), step.mod[:, 2], step.mod[:, 3], step.mod[:, 4],
                                   step.cs, step.cp, res_out=rv(step.rout), norm_out=rv(step.aout), eps=w.eps)

    fshape = frames_shape(scale)
    frames_in = W.frames_input(fshape, seed=step.w.seed).to(step.q.device)
    frames_out = torch.empty(fshape[0:1] + fshape[2:] + fshape[1:2], dtype=torch.uint8, device=step.q.device)

    def frames():
        d.dit_frames_to_u8(frames_in, layout="bthwc", out=frames_out)

    out = {}
    for name, fn in (("gated_residual_adaln", fused), ("frames_to_u8", frames)):
        for _ in range(warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize(device)
        for a, b in ev:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize(device)
        out[name] = statistics.fmean(a.elapsed_time(b) for a, b in ev)
    return out


def host_inputs(w: W.Workload) -> dict:
    qk = W.qk_inputs(w)
    adaln = W.adaln_inputs(w)
    res = W.residual_inputs(w)
    res["mod"] = adaln["mod"]
    return {"qk": qk, "adaln": adaln, "res": res, "swiglu": W.swiglu_inputs(w)}


def time_device(step: Step, steps: int, warmup: int, device):
    """K steps timed bare (the headline: nothing between the kernels but the
    kernels and one CUDA event per step boundary, which gives each step's
    time), then K more with CUDA events around every op for the per-op
    figures (those events sit between the kernels, so they stay out of the
    headline pass).  Returns (elapsed ms of the K headline steps, per-step ms,
    {op: per-launch ms}, host time window of the headline pass)."""
    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        step.run()
    marks = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    barrier()
    torch.cuda.synchronize(device)
    t_host0 = time.time()
    marks[0].record(stream)
    for i in range(steps):
        step.run()
        marks[i + 1].record(stream)
    torch.cuda.synchronize(device)
    t_host1 = time.time()
    barrier()
    elapsed_ms = marks[0].elapsed_time(marks[-1])
    step_ms = [marks[i].elapsed_time(marks[i + 1]) for i in range(steps)]
    per_op = {op: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)] for op in OPS}
    for i in range(steps):
        step.run({op: per_op[op][i] for op in OPS})
    torch.cuda.synchronize(device)
    op_ms = {op: [a.elapsed_time(b) for a, b in per_op[op]] for op in OPS}
    return elapsed_ms, step_ms, op_ms, (t_host0, t_host1)


def time_graph(step: Step, steps: int, warmup: int, device) -> float:
    """The same step captured once in a CUDA graph and replayed `steps` times
    (the library's calls only enqueue work, so they capture as they are):
    mean ms per replay, for comparison with the eagerly launched step."""
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(stream):
        for _ in range(2):
            step.run()  # warm the launch paths on the capture stream
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step.run()
    for _ in range(warmup):
        graph.replay()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(device)
    start.record()
    for _ in range(steps):
        graph.replay()
    end.record()
    torch.cuda.synchronize(device)
    barrier()
    ms = start.elapsed_time(end) / steps
    del graph
    return ms


def time_e2e(sets, steps: int, warmup: int, device):
    """The same step through the public API for a caller whose data lives in
    pinned host memory: every step uploads each op's inputs, runs the op and
    downloads its outputs, all inside the timed region.  Uploads, kernels and
    downloads run on three streams ordered by events, so the two copy
    directions overlap each other and the kernels; two device buffer sets
    alternate between steps (q and k are updated in place).  Returns None on
    every rank when any rank cannot pin its host buffers."""
    try:
        h_in = {op: [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in sets[0].op_inputs(op)]
                for op in OPS}
        h_out = {op: [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in sets[0].op_outputs(op)]
                 for op in OPS}
        pinned = 1.0
    except RuntimeError:  # the host could not pin the step's buffers
        h_in = h_out = None
        pinned = 0.0
    # every rank takes the same collective steps: all time the leg, or none does
    if reduce_max(1.0 - pinned, torch.device("cuda", torch.cuda.current_device())) > 0.0:
        return None
    for op in OPS:
        for h, d in zip(h_in[op], sets[0].op_inputs(op)):
            h.copy_(d)
    h2d = sum(h.numel() * h.element_size() for op in OPS for h in h_in[op])
    d2h = sum(h.numel() * h.element_size() for op in OPS for h in h_out[op])
    s_up, s_run, s_down = (torch.cuda.Stream(device) for _ in range(3))
    free = [None] * len(sets)

    def one(k):
        slot = k % len(sets)
        st = sets[slot]
        ready, done = {}, {}
        with torch.cuda.stream(s_up):
            if free[slot] is not None:
                s_up.wait_event(free[slot])
            for op in OPS:
                for d, h in zip(st.op_inputs(op), h_in[op]):
                    d.copy_(h, non_blocking=True)
                ready[op] = torch.cuda.Event()
                ready[op].record(s_up)
        with torch.cuda.stream(s_run):
            for op in OPS:
                s_run.wait_event(ready[op])
                st.run_op(op)
                done[op] = torch.cuda.Event()
                done[op].record(s_run)
        with torch.cuda.stream(s_down):
            for op in OPS:
                s_down.wait_event(done[op])
                for h, d in zip(h_out[op], st.op_outputs(op)):
                    h.copy_(d, non_blocking=True)
            free[slot] = torch.cuda.Event()
            free[slot].record(s_down)

    for k in range(warmup):
        one(k)
    barrier()
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_up)
    s_run.wait_stream(s_up)
    s_down.wait_stream(s_up)
    for k in range(steps):
        one(k)
    s_down.wait_stream(s_run)
    s_down.wait_stream(s_up)
    end.record(s_down)
    torch.cuda.synchronize(device)
    barrier()
    return start.elapsed_time(end), h2d, d2h


# ------------------------------------------------------------ CPU oracle

class OracleRunner:
    """The CPU oracle over a row sample of the workload (the same four ops)."""

    def __init__(self, w: W.Workload, host: dict):
        import oracle
        from oracle import build as obuild
        obuild.build()
        self.o = oracle
        self.w = w
        bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
        rv = W.rows_view
        self.q, self.k = bits(rv(host["qk"]["q"])), bits(rv(host["qk"]["k"]))
        self.wq, self.wk = bits(host["qk"]["q_weight"]), bits(host["qk"]["k_weight"])
        self.ax = bits(rv(host["adaln"]["x"]))
        self.mod = np.ascontiguousarray(bits(host["adaln"]["mod"]).reshape(-1))
        self.rx, self.ry = bits(rv(host["res"]["x"])), bits(rv(host["res"]["y"]))
        self.ab = bits(rv(host["swiglu"]["ab"]))
        self.outs = {"q": np.empty_like(self.q), "k": np.empty_like(self.k), "a": np.empty_like(self.ax),
                     "r": np.empty_like(self.rx),
                     "s": np.empty((self.ab.shape[0], w.inner), dtype=np.uint16)}

    def threads(self) -> int:
        return self.o.num_threads()

    def run(self, rows: np.ndarray) -> float:
        """Seconds the four oracle calls take on ``rows``."""
        w, o, C = self.w, self.o, self.w.hidden
        t0 = time.perf_counter()
        o.qk_rmsnorm_rope(self.q, self.k, self.wq, self.wk, w.cu_seqlens, w.cu_seqlens_padded,
                          num_q_heads=w.num_q_heads, num_k_heads=w.num_k_heads, head_dim=w.head_dim,
                          rope_grid=w.rope_grid, sections=w.sections, rope_theta=w.rope_theta, eps=w.eps,
                          rows=rows, q_out=self.outs["q"], k_out=self.outs["k"], pos_offset=w.pos_offsets)
        o.adaln_modulate(self.ax, self.mod, self.mod[C:], w.cu_seqlens, w.cu_seqlens_padded, hidden=C,
                         eps=w.eps, mod_seq_stride=6 * C, rows=rows, out=self.outs["a"])
        o.gated_residual(self.rx, self.ry, self.mod[2 * C:], w.cu_seqlens, w.cu_seqlens_padded, hidden=C,
                         gate_seq_stride=6 * C, rows=rows, out=self.outs["r"])
        o.swiglu(self.ab, self.ab.reshape(-1)[w.inner:], w.cu_seqlens, w.cu_seqlens_padded, inner=w.inner,
                 a_row_stride=2 * w.inner, b_row_stride=2 * w.inner, nrows=self.ab.shape[0], rows=rows,
                 out=self.outs["s"])
        return time.perf_counter() - t0

    def sample(self, n: int, seed: int) -> np.ndarray:
        valid = self.w.valid_rows()
        rng = np.random.default_rng(seed)
        return np.sort(rng.choice(valid, size=min(n, valid.size), replace=False))

    def calibrate(self, budget_s: float, seed: int = 7) -> int:
        """Rows per sample so that one sample takes about budget_s."""
        n = 64
        t = self.run(self.sample(n, seed))
        while t < 0.25 and n < self.w.num_valid:
            n *= 4
            t = self.run(self.sample(n, seed))
        return int(max(16, min(self.w.num_valid, n * budget_s / max(t, 1e-6))))


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w: W.Workload, host: dict, budget_s: float = 12.0, budget_1t_s: float = 5.0) -> dict:
    """The oracle as it stands on a bounded seeded sample of the workload's
    valid tokens: once with OpenMP on every host thread it gets, once with
    one thread."""
    runner = OracleRunner(w, host)
    n = runner.calibrate(budget_s)
    rows = runner.sample(n, seed=11)
    t = runner.run(rows)
    threads = runner.threads()
    runner.o.set_num_threads(1)
    try:
        n1 = runner.calibrate(budget_1t_s)
        rows1 = runner.sample(n1, seed=12)
        t1 = runner.run(rows1)
    finally:
        runner.o.set_num_threads(threads)
    return {"value": rows.size / t, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{rows.size} of {w.num_valid} valid tokens of {w.name} (seeded random rows), "
                      f"all four ops per token, fp64 C oracle, {t:.1f} s on {threads} threads",
            "value_1thread": rows1.size / t1,
            "sample_1thread": f"{rows1.size} seeded random valid tokens, {t1:.1f} s on 1 thread",
            "cpu_model": cpu_model(), "host_threads": os.cpu_count()}


# ------------------------------------------------------------ main

def config_block(w: W.Workload, n: int, split: bool = False, whole: W.Workload = None) -> dict:
    src = whole if whole is not None else w
    cfg = {"workload": src.name, "num_seqs": src.num_seqs, "valid_tokens": src.num_valid,
           "padded_rows": src.num_rows_padded, "lengths": list(src.lengths), "hidden": src.hidden,
           "heads": f"{src.num_q_heads}+{src.num_k_heads}x{src.head_dim}", "inner": src.inner,
           "rope": "3d t/h/w 44/42/42 on 24x42 frames + 1d tail" if src.grids else "1d",
           "ops_per_step": list(OPS),
           "l2": "inputs larger than L2 (each op moves >= 1.4 GB per step vs 126 MB L2)",
           "parallelism": f"dp{n}: every GPU runs its own batch, no collective on the data path"}
    if split:
        cfg["parallelism"] = (f"rows{n}: one batch split by valid tokens over {n} ranks (contiguous, count-"
                              "balanced slices with whole-sequence rotary positions), no collective on the "
                              "data path")
        cfg["rank0_slice"] = {"valid_tokens": w.num_valid, "padded_rows": w.num_rows_padded,
                              "lengths": list(w.lengths), "pos_offset": list(w.pos_offset or ())}
        cfg["l2"] = "per-rank slices; each op's working set per step is larger than L2 at 8 ranks or fewer"
    return cfg


def split_workload(w: W.Workload, rank: int, world: int) -> W.Workload:
    """Rank ``rank``'s slice of one batch split over ``world`` ranks by valid
    tokens (``dit_token_b200.shard``): its sequences' pieces, their padding,
    grids and whole-sequence position offsets.  Every rank draws its slice's
    values from the batch's seed (the timing depends on shapes, not values)."""
    from dit_token_b200.shard import shard_packing
    sh = shard_packing(w.cu_seqlens, w.cu_seqlens_padded, w.rope_grid, rank, world)
    return dataclasses.replace(
        w, name=f"{w.name} rank {rank}/{world}", lengths=tuple(int(v) for v in np.diff(sh.cu_seqlens)),
        padded=tuple(int(v) for v in np.diff(sh.cu_seqlens_padded)),
        grids=None if sh.rope_grid is None else tuple(tuple(int(t) for t in g) for g in sh.rope_grid),
        pos_offset=tuple(int(v) for v in sh.pos_offset), seed=w.seed + 7919 * rank)


def plan(args, rank: int, world: int):
    """(this rank's workload, the whole job's workload, valid tokens per step
    over all ranks, scaling mode)."""
    w0 = W.scaled(W.workload(args.workload, args.seed), args.scale)
    if getattr(args, "split", False):
        return split_workload(w0, rank, world), w0, w0.num_valid, "strong"
    return dataclasses.replace(w0, seed=data_seed(args.seed, rank)), w0, w0.num_valid * world, "weak"


SMALL_SHAPES = ("single_stream", "long_video_slice")
LAUNCH_CHAIN = 8  # buffer sets in --launch-cost's chain (per-rank shapes: 8 x 67-380 MB, beyond the 126 MB L2)


def time_small_shapes(device, seed: int, steps: int = 100, reps: int = 30) -> dict:
    """The four-op step at the per-rank-sized shapes (one rank's slice of the
    long video under an 8-way split, and the single-stream workload): per-step
    times of back-to-back eager steps and of graph replays, against the sum of
    each op timed alone (an L2-evicting read before every launch, median of
    ``reps``)."""
    flush = torch.ones(128 * 1024 * 1024, dtype=torch.float32, device=device)  # 512 MB, 4x L2
    out = {}
    for name in SMALL_SHAPES:
        w = W.workload(name, seed)
        step = Step(w, host_inputs(w), device)
        stream = torch.cuda.current_stream(device)
        for _ in range(5):
            step.run()
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        torch.cuda.synchronize(device)
        marks[0].record(stream)
        for i in range(steps):
            step.run()
            marks[i + 1].record(stream)
        torch.cuda.synchronize(device)
        step_ms = [marks[i].elapsed_time(marks[i + 1]) for i in range(steps)]
        graph_ms = time_graph(step, steps, 5, device)
        alone = {}
        for op in OPS:
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            for a, b in ev:
                flush.sum()  # a read-only pass: the kernel starts on clean L2 lines
                a.record()
                step.run_op(op)
                b.record()
            torch.cuda.synchronize(device)
            alone[op] = statistics.median(a.elapsed_time(b) for a, b in ev)
        abytes = algorithmic_bytes(w)
        peak, _ = measured_peak()
        med = statistics.median(step_ms)
        out[name] = {
            "valid_tokens": w.num_valid, "hidden": w.hidden, "inner": w.inner,
            "step": spread(step_ms), "graph_us_per_step": round(graph_ms * 1e3, 2),
            "tokens_per_s": round(w.num_valid / (med / 1e3), 1),
            "step_hbm_frac": round(sum(abytes.values()) / (med / 1e3) / 1e9 / peak, 4),
            "ops_alone_us": {op: round(v * 1e3, 2) for op, v in alone.items()},
            "ops_alone_frac": {op: round(abytes[op] / (alone[op] / 1e3) / 1e9 / peak, 4) for op in OPS},
            "sum_alone_us": round(sum(alone.values()) * 1e3, 2),
            "step_over_sum_alone": round(med / sum(alone.values()), 4)}
        del step
        torch.cuda.empty_cache()
    return out


def measure(args, w: W.Workload, device, world: int) -> dict:
    """Every GPU measurement of the line, this rank's own numbers (ms)."""
    host = host_inputs(w)
    step = Step(w, host, device)
    sampler = ClockSampler(device.index or 0)
    sampler.start()
    elapsed_ms, step_list, op_lists, (h0, h1) = time_device(step, args.steps, args.warmup, device)
    sampler.stop()
    m = {"elapsed_ms": elapsed_ms, "step_ms": step_list, "op_ms": op_lists, "clocks": sampler.summary(h0, h1)}
    m["next_ms"] = time_next_ops(step, args.steps, args.warmup, device, args.scale)
    m["graph_ms"] = time_graph(step, args.steps, args.warmup, device)
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    # two device buffer sets let consecutive end-to-end steps overlap; the
    # small profiling-size runs (--scale < 1) keep one to stay small
    sets = [step, Step(w, host, device)] if args.scale >= 1.0 else [step]
    m["e2e"] = time_e2e(sets, e2e_steps, min(args.warmup, 3), device)
    m["e2e_steps"] = e2e_steps
    del sets, step
    torch.cuda.empty_cache()
    if world == 1 and not args.no_small_shapes:
        m["small_shapes"] = time_small_shapes(device, args.seed)
    if world == 1 and not args.no_cpu_baseline:
        m["cpu_baseline"] = cpu_baseline(w, host, args.cpu_budget)
    return m


def assemble(args, world: int, w: W.Workload, whole: W.Workload, tokens: int, scaling: str, m: dict,
             device) -> dict:
    """The JSON line from this rank's measurements; every rank takes the same
    collective steps (max over ranks of each time)."""
    max_ms = reduce_max(m["elapsed_ms"], device)
    op_ms_max = {op: reduce_max(statistics.fmean(v), device) for op, v in m["op_ms"].items()}
    next_ms = {k: reduce_max(v, device) for k, v in m["next_ms"].items()}
    graph_ms = reduce_max(m["graph_ms"], device)
    timed_e2e = m["e2e"]
    e2e_steps = m["e2e_steps"]
    if timed_e2e is None:
        e2e = {"value": None, "unit": UNIT,
               "unavailable": "the host could not pin the step's input and output buffers on every rank"}
    else:
        e2e_ms, h2d, d2h = timed_e2e
        e2e_max = reduce_max(e2e_ms, device)
        e2e = {"value": round(tokens * e2e_steps / (e2e_max / 1e3), 1), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "ms_per_step": round(e2e_max / e2e_steps, 3),
               "schedule": "per-op upload / kernel / download on 3 streams, 2 device buffer sets"}
    value = tokens * args.steps / (max_ms / 1e3)
    abytes = algorithmic_bytes(w)
    peak, peak_kind = measured_peak()
    ops = {}
    for op in OPS:
        gbs = abytes[op] / (op_ms_max[op] / 1e3) / 1e9
        ops[op] = {"us": round(op_ms_max[op] * 1e3, 2), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
                   "bytes": abytes[op], "spread": spread(m["op_ms"][op])}
    dom = max(OPS, key=lambda o: op_ms_max[o])
    dom_gbs = abytes[dom] / (op_ms_max[dom] / 1e3) / 1e9
    step_gbs = sum(abytes.values()) / (max_ms / args.steps / 1e3) / 1e9
    fshape = frames_shape(args.scale)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 4), "higher_is_better": True,
        "scaling": scaling, "vs_baseline": None, "dtype": "bf16",
        "arith": "f32 (bf16 tensors, fp32 arithmetic, one rounding per output)",
        "data": "synthetic (seeded N(0,1) activations, 1+N(0,0.02) norm weights, N(0,0.1) modulation)",
        "config": config_block(w, world, split=scaling == "strong", whole=whole),
        "step_gbs": round(step_gbs, 1), "step_hbm_frac": round(step_gbs / peak, 4),
        "step_spread": spread(m["step_ms"]),
        "ops": ops,
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": round(dom_gbs, 1), "peak": peak,
                     "peak_kind": f"{peak_kind} HBM copy bandwidth", "unit": "GB/s",
                     "frac": round(dom_gbs / peak, 4), "traffic": profiled_traffic(dom, w.name),
                     "algorithmic_bytes": abytes[dom]},
        "gpu_launches": len(OPS) * args.steps,
        "next_ops": {
            "gated_residual_adaln": {
                "us": round(next_ms["gated_residual_adaln"] * 1e3, 2),
                "gbs": round(8 * w.hidden * w.num_valid / (next_ms["gated_residual_adaln"] / 1e3) / 1e9, 1),
                "bytes": 8 * w.hidden * w.num_valid,
                "unfused_us": round((op_ms_max["gated_residual"] + op_ms_max["adaln_modulate"]) * 1e3, 2)},
            "frames_to_u8": {
                "workload": f"fp32 {list(fshape)} -> uint8 BTHWC (the pages' 10 s 1344x768 "
                            "request: 243 frames)",
                "us": round(next_ms["frames_to_u8"] * 1e3, 2),
                "gbs": round(5 * math.prod(fshape) / (next_ms["frames_to_u8"] / 1e3) / 1e9, 1),
                "bytes": 5 * math.prod(fshape)},
        },
        "e2e": e2e,
        "graph": {"ms_per_step": round(graph_ms, 4), "steps": args.steps,
                  "note": "the same step captured once in a CUDA graph and replayed; value uses the eager step"},
        "clocks": m["clocks"],
    }
    if "small_shapes" in m:
        line["small_shapes"] = m["small_shapes"]
    if "cpu_baseline" in m:
        line["cpu_baseline"] = m["cpu_baseline"]
    return line


def run_dit(args):
    import torch.distributed as dist
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        # the rank's device first, and the group bound to it (its communicator
        # then lives on this GPU, whatever device the first collective sees)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    from dit_token_b200 import build
    if rank == 0 or world == 1:
        build.build()
    barrier()
    w, whole, tokens, scaling = plan(args, rank, world)
    m = measure(args, w, device, world)
    line = assemble(args, world, w, whole, tokens, scaling, m, device)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return  # the CPU oracle runs once, on rank 0
    w = W.scaled(W.workload(args.workload, args.seed), args.scale)
    host = host_inputs(w)
    runner = OracleRunner(w, host)
    per_step = max(0.5, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    n = runner.calibrate(per_step)
    for i in range(args.warmup):
        runner.run(runner.sample(n, seed=100 + i))
    times = [runner.run(runner.sample(n, seed=1000 + i)) for i in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    sample = (f"each step: {n} of {w.num_valid} valid tokens of {w.name} (seeded random rows), all four ops "
              f"per token, fp64 C oracle")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(w, 1), "impl": "reference",
        "cpu_baseline": {"value": round(value, 2), "unit": UNIT, "cores": runner.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def run_table(args):
    """Per-op table over every workload (markdown on stdout), complementing the
    single JSON line.  Each launch is preceded by a read-only pass over 512 MB
    that evicts L2 (the small workloads would otherwise be served from L2)
    and leaves it holding clean lines -- a write would leave dirty lines
    whose write-back the timed kernel would pay for -- and keeps the GPU busy
    while the next launch is submitted, so the CUDA events around the launch
    see the kernel alone."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from dit_token_b200 import build
    build.build()
    import dit_token_b200 as dit
    peak, kind = measured_peak()
    flush = torch.ones(128 * 1024 * 1024, dtype=torch.float32, device=device)  # 512 MB, 4x L2

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ev:
            flush.sum()  # a read-only pass: L2 ends up holding clean lines
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize(device)
        return statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3  # us

    sampler = ClockSampler(0)
    sampler.start()
    print(f"| workload | op | GPU us | tokens/s | GB/s | % of 8 TB/s | % of {kind} {peak:.0f} GB/s |")
    print("|---|---|---|---|---|---|---|")
    for name in W.WORKLOAD_NAMES:
        w = W.workload(name, args.seed)
        host = host_inputs(w)
        step = Step(w, host, device)
        rv = W.rows_view
        ab = algorithmic_bytes(w)
        ab["gated_residual_adaln"] = 8 * w.hidden * w.num_valid
        fns = {op: (lambda op=op: step.run_op(op)) for op in OPS}
        fns["gated_residual_adaln"] = lambda: dit.dit_gated_residual_adaln(
            rv(step.rx), rv(step.ry), step.mod[:, 2], step.mod[:, 3], step.mod[:, 4], step.cs, step.cp,
            res_out=rv(step.rout), norm_out=rv(step.aout), eps=w.eps)
        for op, fn in fns.items():
            us = timed(fn)
            gbs = ab[op] / (us * 1e-6) / 1e9
            print(f"| {name} | {op} | {us:.1f} | {w.num_valid / (us * 1e-6):.3g} | {gbs:.0f} | "
                  f"{100 * gbs / 8000:.1f} | {100 * gbs / peak:.1f} |", flush=True)
        del step, host, fns
        torch.cuda.empty_cache()
    fin = W.frames_input(W.FRAMES_SHAPE, seed=args.seed).to(device)
    fout = torch.empty((1, 243, 768, 1344, 3), dtype=torch.uint8, device=device)
    us = timed(lambda: dit.dit_frames_to_u8(fin, layout="bthwc", out=fout))
    gbs = 5 * FRAMES_ELEMS / (us * 1e-6) / 1e9
    print(f"| frames 1x3x243x768x1344 | frames_to_u8 (BTHWC) | {us:.1f} | - | {gbs:.0f} | "
          f"{100 * gbs / 8000:.1f} | {100 * gbs / peak:.1f} |", flush=True)
    print(clock_note(sampler), flush=True)


def run_variants(args):
    """Markdown table of the operator variants (fp32 and per-stream modulation
    vectors, rotary layouts, grouped K heads, head_dim 256) on the batched
    varlen and long video workloads, and of Q/K normalization and SwiGLU at
    VAE-like shapes, timed like --table (L2 evicted before every launch,
    median of --steps launches)."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from dit_token_b200 import build
    build.build()
    import dit_token_b200 as dit
    peak, kind = measured_peak()
    flush = torch.ones(128 * 1024 * 1024, dtype=torch.float32, device=device)  # 512 MB, 4x L2
    rv = W.rows_view

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ev:
            flush.sum()  # a read-only pass: L2 ends up holding clean lines
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize(device)
        return statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3  # us

    def row(wname, op, variant, us, nbytes, tokens):
        gbs = nbytes / (us * 1e-6) / 1e9
        print(f"| {wname} | {op} | {variant} | {us:.1f} | {tokens / (us * 1e-6):.3g} | {gbs:.0f} | "
              f"{100 * gbs / peak:.1f} |", flush=True)

    sampler = ClockSampler(0)
    sampler.start()
    print(f"| workload | op | variant | GPU us | tokens/s | GB/s | % of {kind} {peak:.0f} GB/s |")
    print("|---|---|---|---|---|---|---|")
    for name in ("batched_varlen", "long_video"):
        w = W.workload(name, args.seed)
        C, B, n = w.hidden, w.num_seqs, w.num_valid
        step = Step(w, host_inputs(w), device)
        m32 = W.modulation(w, torch.float32).to(device)
        cs2, cp2 = dit.dit_av_stream_seqlens(step.cs, step.cp, step.grid)
        mav = W.modulation_av(w).to(device).view(2 * B, 6, C)
        mods = {"bf16 vectors": (step.mod, step.cs, step.cp), "fp32 vectors": (m32, step.cs, step.cp),
                "per-stream bf16 vectors": (mav, cs2, cp2)}
        for variant, (m, cs, cp) in mods.items():
            row(name, "adaln_modulate", variant, timed(lambda: dit.dit_adaln_modulate(
                rv(step.ax), m[:, 0], m[:, 1], cs, cp, out=rv(step.aout), eps=w.eps)), 4 * C * n, n)
            row(name, "gated_residual", variant, timed(lambda: dit.dit_gated_residual(
                rv(step.rx), rv(step.ry), m[:, 2], cs, cp, out=rv(step.rout))), 6 * C * n, n)
            row(name, "gated_residual_adaln", variant, timed(lambda: dit.dit_gated_residual_adaln(
                rv(step.rx), rv(step.ry), m[:, 2], m[:, 3], m[:, 4], cs, cp, res_out=rv(step.rout),
                norm_out=rv(step.aout), eps=w.eps)), 8 * C * n, n)
        row(name, "av_stream_seqlens", f"{B} requests", timed(lambda: dit.dit_av_stream_seqlens(
            step.cs, step.cp, step.grid, out=(cs2, cp2))), 0, n)
        for mode in ("interleaved", "half", "none"):
            row(name, "qk_rmsnorm_rope", f"{mode} pairs, {w.num_q_heads}x{w.head_dim}",
                timed(lambda: dit.dit_qk_rmsnorm_rope(
                    rv(step.q), rv(step.k), step.wq, step.wk, step.cs, step.cp, num_q_heads=w.num_q_heads,
                    num_k_heads=w.num_k_heads, head_dim=w.head_dim, rope_grid=step.grid, sections=w.sections,
                    rope_theta=w.rope_theta, eps=w.eps, rope_mode=mode)), 8 * C * n, n)
        # grouped K heads (a fifth of the q heads), and head_dim 256 over the same q and k widths
        hk = max(1, w.num_q_heads // 5)
        kq = rv(step.k)[:, : hk * w.head_dim]
        row(name, "qk_rmsnorm_rope", f"GQA {w.num_q_heads}q/{hk}k x{w.head_dim}", timed(
            lambda: dit.dit_qk_rmsnorm_rope(
                rv(step.q), kq, step.wq, step.wk, step.cs, step.cp, num_q_heads=w.num_q_heads, num_k_heads=hk,
                head_dim=w.head_dim, rope_grid=step.grid, sections=w.sections, rope_theta=w.rope_theta,
                eps=w.eps)), 4 * (w.num_q_heads + hk) * w.head_dim * n, n)
        w256 = torch.ones(256, dtype=torch.bfloat16, device=device)
        for mode, sec in (("half", (88, 84, 84)), ("none", (0, 0, 0))):
            row(name, "qk_rmsnorm_rope", f"{mode} pairs, {C // 256}x256", timed(
                lambda: dit.dit_qk_rmsnorm_rope(
                    rv(step.q), rv(step.k), w256, w256, step.cs, step.cp, num_q_heads=C // 256,
                    num_k_heads=C // 256, head_dim=256, rope_grid=step.grid, sections=sec,
                    rope_theta=w.rope_theta, eps=w.eps, rope_mode=mode)), 8 * C * n, n)
        del step, mods, m32, mav
        torch.cuda.empty_cache()

    # VAE-like shapes (the pages reuse the fused Q/K norm and SwiGLU in the VAE
    # decoder and give no shapes): one sequence of 2^20 tokens, 512 channels as
    # 8 heads of 64 without rotation, SwiGLU inner 512.  Values N(0, 1) drawn on
    # the device (only the timing is of interest here).
    n = 1 << 20
    gen = torch.Generator(device=device).manual_seed(args.seed)
    cs = torch.tensor([0, n], dtype=torch.int32, device=device)
    q = torch.randn(n, 512, generator=gen, device=device).to(torch.bfloat16)
    k = torch.randn(n, 512, generator=gen, device=device).to(torch.bfloat16)
    w64 = torch.ones(64, dtype=torch.bfloat16, device=device)
    row("vae 1x1048576", "qk_rmsnorm_rope", "none pairs, 8x64", timed(lambda: dit.dit_qk_rmsnorm_rope(
        q, k, w64, w64, cs, cs, num_q_heads=8, num_k_heads=8, head_dim=64, rope_mode="none")), 8 * 512 * n, n)
    del q, k
    ab = torch.randn(n, 1024, generator=gen, device=device).to(torch.bfloat16)
    out = torch.empty(n, 512, dtype=torch.bfloat16, device=device)
    row("vae 1x1048576", "swiglu", "inner 512", timed(lambda: dit.dit_swiglu(
        ab[:, :512], ab[:, 512:], cs, cs, out=out)), 6 * 512 * n, n)
    del ab, out
    torch.cuda.empty_cache()
    print(clock_note(sampler), flush=True)


def run_host_overhead(args):
    """Host time per call of every entry point on the tiny workload: 1,000
    calls back to back with no synchronization (the GPU queue absorbs them),
    once through the Python binding and once as a bare C-ABI call through
    ctypes with its arguments prepared beforehand (what a C caller pays, plus
    ctypes' own few hundred ns).  Markdown on stdout."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from dit_token_b200 import build
    build.build()
    import ctypes
    import dit_token_b200 as dit
    L = dit.library()
    w = W.workload("tiny", args.seed)
    step = Step(w, host_inputs(w), device)
    rv = W.rows_view
    C, I = w.hidden, w.inner
    st = torch.cuda.current_stream(device).cuda_stream
    cs, cp = step.cs.data_ptr(), step.cp.data_ptr()
    B, R = w.num_seqs, w.num_rows_padded
    q, k, ax, ao = rv(step.q), rv(step.k), rv(step.ax), rv(step.aout)
    rx, ry, ro = rv(step.rx), rv(step.ry), rv(step.rout)
    ab, so = rv(step.ab), rv(step.sout)
    m = step.mod
    norm = torch.empty_like(ro)
    flag = torch.empty(2, dtype=torch.int32, device=device)
    cs2 = torch.empty(2 * B + 1, dtype=torch.int32, device=device)
    cp2 = torch.empty_like(cs2)
    grid1 = torch.tensor([[1, 10, 20]], dtype=torch.int32, device=device)
    frames = W.frames_input((1, 3, 2, 16, 32)).to(device)
    fout = torch.empty((1, 2, 16, 32, 3), dtype=torch.uint8, device=device)
    qs, ks = q.stride(0), k.stride(0)
    hd = w.head_dim
    raw = {
        "dit_qk_rmsnorm_rope": (L.dit_qk_rmsnorm_rope, (
            q.data_ptr(), qs, k.data_ptr(), ks, step.wq.data_ptr(), step.wk.data_ptr(), cs, cp, B, R,
            w.num_q_heads, w.num_k_heads, hd, None, 0, 0, 0, 10000.0, 1e-6, st)),
        "dit_adaln_modulate": (L.dit_adaln_modulate, (
            ax.data_ptr(), C, ao.data_ptr(), C, m[:, 0].data_ptr(), m[:, 1].data_ptr(), 6 * C, cs, cp, B, R, C,
            1e-6, st)),
        "dit_gated_residual": (L.dit_gated_residual, (
            rx.data_ptr(), C, ry.data_ptr(), C, m[:, 2].data_ptr(), 6 * C, ro.data_ptr(), C, cs, cp, B, R, C, st)),
        "dit_swiglu": (L.dit_swiglu, (
            ab.data_ptr(), 2 * I, ab[:, I:].data_ptr(), 2 * I, so.data_ptr(), I, cs, cp, B, R, I, st)),
        "dit_gated_residual_adaln": (L.dit_gated_residual_adaln, (
            rx.data_ptr(), C, ry.data_ptr(), C, m[:, 2].data_ptr(), 6 * C, m[:, 3].data_ptr(), m[:, 4].data_ptr(),
            6 * C, ro.data_ptr(), C, norm.data_ptr(), C, cs, cp, B, R, C, 1e-6, st)),
        "dit_validate_seqlens": (L.dit_validate_seqlens, (cs, cp, B, R, flag.data_ptr(), st)),
        "dit_av_stream_seqlens": (L.dit_av_stream_seqlens, (
            cs, cp, grid1.data_ptr(), None, B, cs2.data_ptr(), cp2.data_ptr(), st)),
        "dit_frames_to_u8": (L.dit_frames_to_u8, (
            ctypes.c_void_p(frames.data_ptr()), 1, 3, 2, 16, 32, 0, ctypes.c_void_p(fout.data_ptr()), st)),
    }
    binding = {
        "dit_qk_rmsnorm_rope": lambda: step.run_op("qk_rmsnorm_rope"),
        "dit_adaln_modulate": lambda: step.run_op("adaln_modulate"),
        "dit_gated_residual": lambda: step.run_op("gated_residual"),
        "dit_swiglu": lambda: step.run_op("swiglu"),
        "dit_gated_residual_adaln": lambda: dit.dit_gated_residual_adaln(
            rx, ry, m[:, 2], m[:, 3], m[:, 4], step.cs, step.cp, res_out=ro, norm_out=norm, eps=w.eps),
        "dit_validate_seqlens": lambda: dit.dit_validate_seqlens(step.cs, step.cp, R, flag=flag),
        "dit_av_stream_seqlens": lambda: dit.dit_av_stream_seqlens(step.cs, step.cp, grid1, out=(cs2, cp2)),
        "dit_frames_to_u8": lambda: dit.dit_frames_to_u8(frames, layout="bthwc", out=fout),
    }
    n = 1000
    print("| entry point | host us per call, C ABI via ctypes | host us per call, Python binding |")
    print("|---|---|---|")
    for name, (fn, a) in raw.items():
        for _ in range(20):
            assert fn(*a) == 0, name
        torch.cuda.synchronize(device)
        t0 = time.perf_counter()
        for _ in range(n):
            fn(*a)
        t1 = time.perf_counter()
        torch.cuda.synchronize(device)
        bfn = binding[name]
        for _ in range(20):
            bfn()
        torch.cuda.synchronize(device)
        t2 = time.perf_counter()
        for _ in range(n):
            bfn()
        t3 = time.perf_counter()
        torch.cuda.synchronize(device)
        print(f"| {name} | {(t1 - t0) / n * 1e6:.2f} | {(t3 - t2) / n * 1e6:.2f} |", flush=True)


def run_launch_cost(args):
    """What one launch costs when timed alone, and what the same call costs
    inside a chain: device time between two CUDA events around the call(s),
    after a read-only pass over 512 MB (clean L2), median of --steps.  Rows:
    nothing between the events, a one-element torch fill, the library's
    smallest kernel, and every op of the tiny and per-rank-sized workloads.
    The chain runs the op on CHAIN separate buffer sets back to back (more
    bytes than L2 holds), so each call after the first reads from HBM and
    writes back its predecessor's dirty lines, as in a stream of ops; the
    per-call cost in the chain is (chain - once) / (CHAIN - 1).  The library
    loaded is the in-tree one, or DIT_TOKEN_LIB (e.g. a build with --define
    DIT_PDL=0)."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from dit_token_b200 import build
    build.build()
    import dit_token_b200 as dit
    peak, kind = measured_peak()
    flush = torch.ones(128 * 1024 * 1024, dtype=torch.float32, device=device)  # 512 MB, 4x L2

    host_us = []

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        host_us.clear()
        for a, b in ev:
            flush.sum()  # a read-only pass: L2 ends up holding clean lines
            # about 0.5 ms of one spinning thread: the host has queued every
            # call of the chain before the first event, so the GPU never
            # waits for the Python side between them
            torch.cuda._sleep(1_000_000)
            a.record()
            t0 = time.perf_counter()
            fn()
            host_us.append((time.perf_counter() - t0) * 1e6)
            b.record()
        torch.cuda.synchronize(device)
        return statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3  # us

    sampler = ClockSampler(0)
    sampler.start()
    n = LAUNCH_CHAIN
    print(f"library: {dit.LIB_PATH}")
    print(f"| workload | call | once us | chain of {n} us | host us to queue the chain | per call in the chain us | "
          f"GB/s in the chain | % of {kind} {peak:.0f} GB/s |")
    print("|---|---|---|---|---|---|---|---|")
    one = torch.zeros(1, device=device)
    print(f"| - | nothing | {timed(lambda: None):.2f} | - | - | - | - | - |")
    print(f"| - | torch fill, 1 element | {timed(lambda: one.fill_(1.0)):.2f} | - | - | - | - | - |")
    cs = torch.tensor([0, 100, 200], dtype=torch.int32, device=device)
    grid = torch.tensor([[2, 5, 5], [1, 2, 3]], dtype=torch.int32, device=device)
    outs = [(torch.empty(5, dtype=torch.int32, device=device), torch.empty(5, dtype=torch.int32, device=device))
            for _ in range(n)]
    av = [lambda o=o: dit.dit_av_stream_seqlens(cs, cs, grid, out=o) for o in outs]
    t1, tn = timed(av[0]), timed(lambda: [f() for f in av])
    print(f"| - | dit_av_stream_seqlens, 2 sequences | {t1:.2f} | {tn:.2f} | {statistics.median(host_us):.1f} | "
          f"{(tn - t1) / (n - 1):.2f} | - | - |", flush=True)
    for name in ("tiny",) + SMALL_SHAPES:
        w = W.workload(name, args.seed)
        host = host_inputs(w)
        sets = [Step(w, host, device) for _ in range(n)]
        ab = algorithmic_bytes(w)
        for op in OPS:
            t1 = timed(lambda: sets[0].run_op(op))
            tn = timed(lambda: [st.run_op(op) for st in sets])
            per = (tn - t1) / (n - 1)
            gbs = ab[op] / (per * 1e-6) / 1e9
            print(f"| {name} | {op} | {t1:.2f} | {tn:.2f} | {statistics.median(host_us):.1f} | {per:.2f} | "
                  f"{gbs:.0f} | {100 * gbs / peak:.1f} |", flush=True)
        del sets, host
        torch.cuda.empty_cache()
    print(clock_note(sampler), flush=True)


def run_profile_op(args):
    """One operator alone, at the workload's full shape, with only its own
    buffers on the device (adaLN on batched varlen: 2 x 718 MB): W + K
    launches back to back, then a synchronize.  For a profiler capture of a
    single full-size launch (e.g. ncu -k regex:adaln_ -s W -c 1)."""
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from dit_token_b200 import build
    build.build()
    w = W.workload(args.workload, args.seed)
    op = args.profile_op
    builders = {"qk_rmsnorm_rope": lambda: {"qk": W.qk_inputs(w)},
                "adaln_modulate": lambda: {"adaln": W.adaln_inputs(w)},
                "gated_residual": lambda: {"res": W.residual_inputs(w)},
                "swiglu": lambda: {"swiglu": W.swiglu_inputs(w)}}
    host = builders[op]()

    class OneOp(Step):
        def __init__(self):
            import dit_token_b200 as dit
            self.dit, self.w = dit, w
            self.cs = torch.from_numpy(w.cu_seqlens).to(device)
            self.cp = torch.from_numpy(w.cu_seqlens_padded).to(device)
            self.grid = None if w.rope_grid is None else torch.from_numpy(w.rope_grid).to(device)
            self.pos_offset = None if w.pos_offset is None else torch.from_numpy(w.pos_offsets).to(device)
            rv = W.rows_view
            self.v = {}
            if "qk" in host:
                self.q, self.k = host["qk"]["q"].to(device), host["qk"]["k"].to(device)
                self.wq, self.wk = host["qk"]["q_weight"].to(device), host["qk"]["k_weight"].to(device)
                self.v.update(q=rv(self.q), k=rv(self.k))
            if "adaln" in host:
                ax, ao, mod = (host["adaln"][k].to(device) for k in ("x", "out", "mod"))
                self.v.update(ax=rv(ax), aout=rv(ao), shift=mod[:, 0], scale=mod[:, 1])
            if "res" in host:
                rx, ry, ro, mod = (host["res"][k].to(device) for k in ("x", "y", "out", "mod"))
                self.v.update(rx=rv(rx), ry=rv(ry), rout=rv(ro), gate=mod[:, 2])
            if "swiglu" in host:
                ab, so = host["swiglu"]["ab"].to(device), host["swiglu"]["out"].to(device)
                self.v.update(a=rv(ab)[:, : w.inner], b=rv(ab)[:, w.inner:], sout=rv(so))

    one = OneOp()
    for _ in range(args.warmup + args.steps):
        one.run_op(op)
    torch.cuda.synchronize(device)
    print(f"{op} on {w.name}: {args.warmup + args.steps} launches", flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("dit", "reference"), default="dit")
    ap.add_argument("--workload", default="batched_varlen", choices=W.WORKLOAD_NAMES)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--scale", type=float, default=1.0,
                    help="scale every sequence's valid length (a smaller batch of the same shapes, "
                         "e.g. for profiling); the JSON names the scaled workload")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-small-shapes", action="store_true",
                    help="skip the step timing at the per-rank-sized shapes (single_stream, long_video_slice)")
    ap.add_argument("--split", action="store_true",
                    help="with --gpus N: the ranks split ONE batch by rows (strong scaling) instead of each "
                         "running its own batch (weak scaling, the default)")
    ap.add_argument("--table", action="store_true",
                    help="print a per-op markdown table over every workload instead of the JSON line")
    ap.add_argument("--variants", action="store_true",
                    help="print a markdown table of the operator variants instead of the JSON line")
    ap.add_argument("--host-overhead", action="store_true",
                    help="print the host time per call of every entry point (tiny workload, no sync)")
    ap.add_argument("--launch-cost", action="store_true",
                    help="print the device time of one call alone and per call in a chain (tiny and "
                         "per-rank sized workloads) instead of the JSON line")
    ap.add_argument("--profile-op", choices=OPS,
                    help="launch only this operator, W + K times on the workload with its own buffers "
                         "(for a profiler capture of one full-size launch)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, _, _ = dist_env()
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 must be launched with torch.distributed.run (one rank per GPU)")
    if args.profile_op:
        run_profile_op(args)
    elif args.host_overhead:
        run_host_overhead(args)
    elif args.launch_cost:
        run_launch_cost(args)
    elif args.table:
        run_table(args)
    elif args.variants:
        run_variants(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_dit(args)


if __name__ == "__main__":
    main()
