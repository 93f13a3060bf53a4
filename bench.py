#!/usr/bin/env python
"""Benchmark of libm3ssd on one node: scan Mtokens/s (forward, L = 4096) and
decode steps/s, each against the B200 HBM roofline, plus an end-to-end figure
through host buffers and the fp64 CPU oracle as a reported baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one m3ssd_fwd over the full Mamba-3 SISO workload (b8 L4096 H32 P64
N128, bf16 X/B/C, fp32 logdecay/beta/gamma/theta/h0, every optional input
present), i.e. one pass of every forward stage: decay and angle cumsums,
rotation, the fused trapezoid intra-chunk products, the chunk-state update,
the inter-chunk state walk and the state-to-output product.  Inputs are
synthetic and seeded; they are resident in HBM when the timed region starts and
larger than L2 (583 MB of algorithmic traffic per step), so no flush is needed.
With N > 1 (torchrun, one process per GPU) every rank runs its own batch
(weak scaling, no collective on the data path); time is the max over ranks.

The decode figure (b256 H32 P64 N128 fp32 cache after a 512-token prefill)
replays one CUDA graph of 1000 m3ssd_step calls.  Side figures in the same line:
MIMO rank-4 decode, the Mamba-3 SISO block at d_model 1024, the backward on the
forward's workload, and the forward on the ssd and long workloads, each with
its own roofline.

Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from selective_state_space_m3ssd_b200.synth import (  # noqa: E402
    DECODE_PREFILL, DECODE_STEPS, MIMO_WORKLOADS, WORKLOADS, make_inputs, make_mimo_inputs,
    rank_workload, slice_inputs)

METRIC = "scan Mtokens/s (fwd, L=4096)"
UNIT = "Mtokens/s"
FWD_KEY = "siso"
PROFILES = os.path.join(ROOT, "profiles")
_CSRC = os.path.join(ROOT, "selective_state_space_m3ssd_b200", "csrc")
# the sources a kernel is built from (a traffic record holds while they are unchanged)
CHUNK_SRC = [os.path.join(_CSRC, f) for f in ("fwd_chunk.cu", "chunk_common.cuh", "tc5.cuh")]
STEP_SRC = [os.path.join(_CSRC, "step.cu")]


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def nbytes(*ts) -> int:
    return sum(t.numel() * t.element_size() for t in ts if t is not None)


def max_over_ranks(ms: float, dev) -> float:
    """The slowest rank's time (ms) when several ranks run, else ``ms``: every
    multi-rank figure is the max over ranks, on the device's own process group."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def src_sha(paths) -> str:
    h = hashlib.sha256()
    for path in ([paths] if isinstance(paths, str) else paths):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(name: str, src: str):
    """DRAM bytes per launch from a committed ncu summary, only while the
    kernel source is the one the counters were taken on."""
    p = os.path.join(PROFILES, f"traffic_{name}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_sha256_16") != src_sha(src):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle sampling in the background during a region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self._t.join(timeout=2)
        return False

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        busy = [s for s in sm if mx and s >= 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# CPU oracle baseline (reported, not the target)
# ----------------------------------------------------------------------------

def oracle_sample(inp_cpu: dict, npairs: int):
    """Run the fp64 oracle on the first ``npairs`` (b, h) sequences of the
    workload (full length each) and return (token-heads, seconds, threads)."""
    import oracle
    b, L, H, P = inp_cpu["X"].shape
    threads = oracle.default_threads()
    pairs = [(k // H, k % H) for k in range(npairs)]
    by_b: dict[int, list[int]] = {}
    for bi, hi in pairs:
        by_b.setdefault(bi, []).append(hi)
    t0 = time.perf_counter()
    for bi, heads in by_b.items():
        sub = slice_inputs(inp_cpu, b=bi, heads=heads)
        oracle.oracle_fwd(**sub, nthreads=threads)
    dt = time.perf_counter() - t0
    return npairs * L, dt, threads


def cpu_baseline(inp_cpu: dict, target_s: float = 10.0) -> dict:
    b, L, H, P = inp_cpu["X"].shape
    import oracle
    threads = oracle.default_threads()
    n0 = min(b * H, max(1, threads))
    th, dt, _ = oracle_sample(inp_cpu, n0)
    n1 = int(min(b * H, max(n0, n0 * target_s / max(dt, 1e-3))))
    if n1 > n0:
        th, dt, _ = oracle_sample(inp_cpu, n1)
    else:
        n1 = n0
    tokens = th / H
    return {"value": tokens / dt / 1e6, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{n1} of {b * H} (b,h) sequences of the workload, full length L={L} "
                      f"({th} token-heads, {dt:.1f} s, fp64 C loop, {threads} threads)"}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def fwd_config(w) -> dict:
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads,
            "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups, "chunk": 64,
            "x_dtype": w.dtype, "state_dtype": "f32", "global_batch": None,
            "l2": "inputs larger than L2 (no flush needed)"}


def fwd_launches_per_call(w, dev, chunk=0) -> int:
    """Kernel launches of one m3ssd_fwd call: three when the chunked bf16 forward
    splits the sequences into segments (segment pass, combine, chunk walk), else
    one."""
    import selective_state_space_m3ssd_b200 as m3
    if w.dtype != "bf16" or w.dstate != 128 or w.headdim != 64 or chunk not in (0, 64):
        return 1
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return 3 if m3.fwd_split_plan(w.batch, w.seqlen, w.nheads, sms)[0] > 1 else 1


def split_of(w, dev):
    """(segments, chunks per segment) of the forward's sequence split on this device."""
    import selective_state_space_m3ssd_b200 as m3
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    return list(m3.fwd_split_plan(w.batch, w.seqlen, w.nheads, sms))


def bench_forward(w, dev, steps, warmup, world, rank):
    import selective_state_space_m3ssd_b200 as m3
    inp = make_inputs(w)
    d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
    hT = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, dtype=torch.float32, device=dev)
    call = m3.PreparedFwd(d["X"], d["logdecay"], d["beta"], d["gamma"], d["B"], d["C"],
                          d["theta"], d["D"], d["h0"], hT=hT)
    algo_bytes = nbytes(*(d[k] for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta",
                                        "D", "h0")), call.Y, hT)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    if world > 1:
        ms = max_over_ranks(ms, dev)
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    return {"ms_total": ms, "ms_per_step": ms / steps, "algo_bytes": algo_bytes, "inp": inp,
            "dev_inputs": d, "call": call, "launches": steps * fwd_launches_per_call(w, dev)}


def forward_leg(key, dev, steps, warmup, world, rank, peaks):
    """The forward on another of the scan workloads (its own inputs, HBM roofline
    on its own algorithmic bytes); a side figure, not the headline."""
    w = rank_workload(WORKLOADS[key], rank)
    fw = bench_forward(w, dev, steps, warmup, world, rank)
    achieved = fw["algo_bytes"] / (fw["ms_per_step"] / 1e3) / 1e9
    out = {"metric": "scan Mtokens/s (fwd)",
           "value": w.batch * w.seqlen * world / (fw["ms_per_step"] / 1e3) / 1e6,
           "unit": "Mtokens/s", "ms_per_step": fw["ms_per_step"], "steps": steps,
           "config": dict(fwd_config(w), split=split_of(w, dev)),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                        "algo_bytes_per_launch": fw["algo_bytes"], "traffic": None,
                        "peak_source": peaks["source"]},
           "gpu_launches": fw["launches"]}
    del fw
    torch.cuda.empty_cache()
    return out


def chunk_sweep_leg(dev, steps, warmup, world, rank, peaks):
    """The forward at chunk lengths Q = 64, 128, 256 (m3ssd_dims.chunk) on the long
    and the siso workloads, each with its HBM roofline; a side figure."""
    import selective_state_space_m3ssd_b200 as m3
    out = {}
    launches = 0
    for key in ("long", "siso"):
        w = rank_workload(WORKLOADS[key], rank)
        d = make_inputs(w, device=dev)
        hT = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, dtype=torch.float32, device=dev)
        args = [d[k] for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")]
        rows = {}
        for Q in (64, 128, 256):
            call = m3.PreparedFwd(*args, hT=hT, chunk=Q)
            algo = nbytes(*(a for a in args if a is not None), call.Y, hT)
            stream = torch.cuda.current_stream(dev)
            for _ in range(warmup):
                call()
            torch.cuda.synchronize(dev)
            if world > 1:
                torch.distributed.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                call()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1)
            if world > 1:
                ms = max_over_ranks(ms, dev)
            per = ms / steps
            ach = algo / (per / 1e3) / 1e9
            rows[f"Q{Q}"] = {"ms_per_step": per,
                             "value": w.batch * w.seqlen * world / (per / 1e3) / 1e6,
                             "unit": "Mtokens/s", "frac": ach / peaks["hbm_gbs"]}
            launches += steps * fwd_launches_per_call(w, dev, Q)
            del call
        out[key] = {"workload": w.name, "by_chunk": rows}
        del d, hT, args
        torch.cuda.empty_cache()
    best = min(out["long"]["by_chunk"].items(), key=lambda kv: kv[1]["ms_per_step"])
    return {"metric": "scan Mtokens/s (fwd) by chunk length", "value": best[1]["value"],
            "unit": "Mtokens/s", "ms_per_step": best[1]["ms_per_step"], "best_long": best[0],
            "roofline": {"bound": "hbm", "frac": best[1]["frac"], "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "peak_source": peaks["source"]},
            "sweep": out, "gpu_launches": launches}


def prefill_leg(dev, steps, warmup, world, rank, peaks):
    """The decode workload's 512-token fp32 prefill (m3ssd_fwd on b256 H32 P64
    N128, fp32 X, B, C, Y: the chunked kernel with fp16 high / low tensor-core
    operands), with an HBM roofline on its algorithmic bytes; a side figure."""
    w = rank_workload(WORKLOADS["decode"].with_(seqlen=DECODE_PREFILL), rank)
    fw = bench_forward(w, dev, steps, warmup, world, rank)
    achieved = fw["algo_bytes"] / (fw["ms_per_step"] / 1e3) / 1e9
    out = {"metric": "scan Mtokens/s (fwd, fp32 prefill)",
           "value": w.batch * w.seqlen * world / (fw["ms_per_step"] / 1e3) / 1e6,
           "unit": "Mtokens/s", "ms_per_step": fw["ms_per_step"], "steps": steps,
           "config": dict(fwd_config(w), workload=f"decode workload prefill b{w.batch} "
                          f"L{w.seqlen} H{w.nheads} P{w.headdim} N{w.dstate} fp32"),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                        "algo_bytes_per_launch": fw["algo_bytes"], "traffic": None,
                        "peak_source": peaks["source"]},
           "gpu_launches": fw["launches"]}
    del fw
    torch.cuda.empty_cache()
    return out


def mimo_forward_leg(dev, steps, warmup, world, rank, peaks):
    """The rank-4 MIMO prefill (m3ssd_mimo_fwd, chunked tensor-core kernel) on its
    own inputs, with an HBM roofline on its algorithmic bytes; a side figure."""
    import selective_state_space_m3ssd_b200 as m3
    base, R = MIMO_WORKLOADS["mimo"]
    w = rank_workload(base, rank)
    d = make_mimo_inputs(w, R, dev)
    Y = torch.empty_like(d["X"])
    args = [d[k] for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")]
    hT = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, dtype=torch.float32, device=dev)
    algo_bytes = nbytes(*args, Y, hT)

    def call():
        m3.mimo_fwd(*args, Y=Y)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    if world > 1:
        ms = max_over_ranks(ms, dev)
    per = ms / steps
    achieved = algo_bytes / (per / 1e3) / 1e9
    # the same prefill with fp32 X, B, C, Y (the chunked kernel on fp16 high / low parts)
    for k in ("X", "B", "C"):
        d[k] = d[k].float()
    args32 = [d[k] for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")]
    Y32 = torch.empty_like(d["X"])
    bytes32 = nbytes(*args32, Y32, hT)
    for _ in range(warmup):
        m3.mimo_fwd(*args32, Y=Y32)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(steps):
        m3.mimo_fwd(*args32, Y=Y32)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    per32 = e0.elapsed_time(e1) / steps
    fp32 = {"ms_per_step": per32, "value": w.batch * w.seqlen * world / (per32 / 1e3) / 1e6,
            "unit": "Mtokens/s", "algo_bytes_per_launch": bytes32,
            "frac": bytes32 / (per32 / 1e3) / 1e9 / peaks["hbm_gbs"]}
    del args32, Y32
    out = {"metric": "MIMO scan Mtokens/s (fwd)",
           "value": w.batch * w.seqlen * world / (per / 1e3) / 1e6,
           "unit": "Mtokens/s", "ms_per_step": per, "steps": steps,
           "config": dict(fwd_config(w), rank=R, chunk_tokens=64 // R - 1),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                        "algo_bytes_per_launch": algo_bytes, "traffic": None,
                        "peak_source": peaks["source"]},
           "fp32": fp32,
           "gpu_launches": 2 * steps}
    del d, Y, hT, args
    torch.cuda.empty_cache()
    return out


def bench_e2e(w, dev, steps, warmup, inp_cpu, world):
    """Same metric through host buffers: every step copies all inputs from pinned
    host memory (H2D), calls the C-ABI forward and copies Y and hT back (D2H),
    all inside the timed region.  Steps are pipelined as a streaming user would:
    two device buffer sets, H2D on one stream, the forward on a second, D2H on a
    third, so that step k's forward overlaps step k+1's H2D and step k-1's D2H
    (PCIe copies in both directions at once)."""
    import selective_state_space_m3ssd_b200 as m3
    keys = ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")
    host = {k: (None if inp_cpu[k] is None else inp_cpu[k].pin_memory()) for k in keys}
    sets = []
    for _ in range(2):
        d = {k: (None if host[k] is None else torch.empty_like(host[k], device=dev)) for k in keys}
        hT = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, dtype=torch.float32, device=dev)
        call = m3.PreparedFwd(d["X"], d["logdecay"], d["beta"], d["gamma"], d["B"], d["C"],
                              d["theta"], d["D"], d["h0"], hT=hT)
        Yh = torch.empty(call.Y.shape, dtype=call.Y.dtype).pin_memory()
        hTh = torch.empty(hT.shape, dtype=hT.dtype).pin_memory()
        sets.append({"d": d, "hT": hT, "call": call, "Yh": Yh, "hTh": hTh})
    h2d = nbytes(*(host[k] for k in keys))
    d2h = nbytes(sets[0]["Yh"], sets[0]["hTh"])
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev = lambda: torch.cuda.Event()
    in_done, cmp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [False, False]

    def one(k):
        i = k % 2
        st = sets[i]
        with torch.cuda.stream(s_in):
            if used[i]:
                s_in.wait_event(cmp_done[i])      # the forward of step k-2 read these inputs
            for key in keys:
                if st["d"][key] is not None:
                    st["d"][key].copy_(host[key], non_blocking=True)
            in_done[i].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_done[i])
            if used[i]:
                s_cmp.wait_event(out_done[i])     # the D2H of step k-2 read Y and hT
            st["call"]()
            cmp_done[i].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[i])
            st["Yh"].copy_(st["call"].Y, non_blocking=True)
            st["hTh"].copy_(st["hT"], non_blocking=True)
            out_done[i].record(s_out)
        used[i] = True

    for k in range(warmup):
        one(k)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(steps):
        one(warmup + k)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    if world > 1:
        ms = max_over_ranks(ms, dev)
    tokens = w.batch * w.seqlen * steps * world
    return {"value": tokens / (ms / 1e3) / 1e6, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms / steps,
            "pipelining": "two buffer sets; H2D, forward and D2H on three streams"}


def bench_decode(dev, rank, steps_graph_replays: int, peaks: dict):
    """Prefill 512 tokens with m3ssd_fwd (fp32 path), then replay one CUDA graph
    of 1000 m3ssd_step calls on pre-staged per-step inputs."""
    import selective_state_space_m3ssd_b200 as m3
    w = rank_workload(WORKLOADS["decode"], rank)
    inp = make_inputs(w, device=dev)
    Lp = DECODE_PREFILL
    pre = {k: (None if inp[k] is None else inp[k][:, :Lp].contiguous())
           for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta")}
    Y, hT, cache = m3.fwd(pre["X"], pre["logdecay"], pre["beta"], pre["gamma"], pre["B"],
                          pre["C"], pre["theta"], inp["D"], None, want_cache=True)
    cache["ssm"] = hT
    del Y, pre
    steps = {k: (None if inp[k] is None else inp[k][:, Lp:].transpose(0, 1).contiguous())
             for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta")}
    D = inp["D"]
    del inp
    ys = torch.empty_like(steps["X"])
    torch.cuda.synchronize(dev)

    def run_steps():
        for t in range(DECODE_STEPS):
            m3.step(cache, steps["X"][t], steps["logdecay"][t], steps["beta"][t],
                    steps["gamma"][t], steps["B"][t], steps["C"][t], steps["theta"][t], D,
                    y_t=ys[t])

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        run_steps()  # warm-up outside the graph
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_steps()
    torch.cuda.synchronize(dev)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps_graph_replays):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    nsteps = DECODE_STEPS * steps_graph_replays
    ms_step = ms / nsteps
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    f = 4
    step_bytes = (2 * b * H * N * P * f          # ssm read + write
                  + 2 * b * H * (N // 2) * f     # angle read + write
                  + 2 * b * H * P * f            # x_prev read + write
                  + 2 * b * G * N * f            # b_prev read + write
                  + b * H * P * f                # x_t
                  + b * H * (N // 2) * f         # theta_t
                  + 2 * b * G * N * f            # B_t, C_t
                  + 3 * b * H * f + H * f        # logdecay_t, beta_t, gamma_t, D
                  + b * H * P * f)               # y_t
    achieved = step_bytes / (ms_step / 1e3) / 1e9
    del g
    return {"metric": "decode steps/s", "value": 1e3 / ms_step, "unit": "steps/s",
            "ms_per_step": ms_step, "graph_steps": nsteps,
            "config": {"workload": w.name, "batch": b, "nheads": H, "headdim": P, "dstate": N,
                       "prefill": Lp, "steps_per_graph": DECODE_STEPS, "dtype": "f32"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "peak_source": peaks["source"],
                         "traffic": recorded_traffic("step_decode", STEP_SRC),
                         "algo_bytes_per_step": step_bytes,
                         "note": "per step = step kernel + b_prev update kernel (2 launches)"},
            "gpu_launches": 2 * nsteps}


def bench_mimo_decode(dev, rank, peaks: dict, R: int = 4, nsteps: int = 100, replays: int = 3):
    """MIMO rank-R decode: one CUDA graph of ``nsteps`` m3ssd_mimo_step calls on
    pre-staged synthetic per-step inputs of the decode workload's shape (fp32
    cache and inputs), replayed ``replays`` times."""
    import selective_state_space_m3ssd_b200 as m3
    w = rank_workload(WORKLOADS["decode"], rank)
    b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
    gen = torch.Generator(device=dev).manual_seed(w.seed + 17)
    z = dict(device=dev, dtype=torch.float32)
    cache = m3.new_mimo_cache(b, H, P, N, G, R, dev)
    cache["ssm"].normal_(0, 0.3, generator=gen)
    xs = torch.randn(nsteps, b, H, P, R, generator=gen, **z)
    Bs = torch.randn(nsteps, b, G, N, R, generator=gen, **z) / N ** 0.5
    Cs = torch.randn(nsteps, b, G, N, R, generator=gen, **z) / N ** 0.5
    ths = torch.randn(nsteps, b, H, N // 2, generator=gen, **z) * 0.05
    lds = -torch.rand(nsteps, b, H, generator=gen, **z) * 0.5
    bes = torch.rand(nsteps, b, H, generator=gen, **z) * 0.3
    gas = torch.rand(nsteps, b, H, generator=gen, **z) * 0.5
    D = torch.randn(H, generator=gen, **z)
    ys = torch.empty_like(xs)

    def run_steps():
        for t in range(nsteps):
            m3.mimo_step(cache, xs[t], lds[t], bes[t], gas[t], Bs[t], Cs[t], ths[t], D, y_t=ys[t])

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        run_steps()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_steps()
    g.replay()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(replays):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_step = e0.elapsed_time(e1) / (nsteps * replays)
    f = 4
    step_bytes = (2 * b * H * N * P * f + 2 * b * H * (N // 2) * f + 2 * b * H * P * R * f
                  + 2 * b * G * N * R * f + b * H * P * R * f + b * H * (N // 2) * f
                  + 2 * b * G * N * R * f + 3 * b * H * f + H * f + b * H * P * R * f)
    achieved = step_bytes / (ms_step / 1e3) / 1e9
    del g
    return {"metric": "mimo decode steps/s", "value": 1e3 / ms_step, "unit": "steps/s",
            "ms_per_step": ms_step, "graph_steps": nsteps * replays,
            "config": {"workload": f"MIMO rank-{R} decode b{b} H{H} P{P} N{N} fp32",
                       "batch": b, "nheads": H, "headdim": P, "dstate": N, "rank": R,
                       "dtype": "f32"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "peak_source": peaks["source"], "traffic": None,
                         "algo_bytes_per_step": step_bytes,
                         "flops_per_step": 2 * 3 * R * b * H * N * P,
                         "note": "per step = MIMO step kernel + b_prev update kernel (2 launches)"},
            "gpu_launches": 2 * nsteps * replays}


def bench_block(dev, rank, peaks: dict, steps: int = 5, warmup: int = 3):
    """The Mamba-3 SISO block forward (m3ssd_block_fwd: in_proj, prep, scan, gate,
    out_proj) at model size d_model 1024, b8 L4096, random-init weights;
    inputs and weights resident in HBM (their sizes exceed L2)."""
    import selective_state_space_m3ssd_b200 as m3
    from selective_state_space_m3ssd_b200.synth import BLOCKS, make_block
    s = BLOCKS["model"].with_(seed=BLOCKS["model"].seed + 7919 * rank)
    u, wts = make_block(s, device=dev)
    out = torch.empty_like(u)
    dims = m3.BlockDims(s.batch, s.seqlen, s.d_model, s.nheads, s.headdim, s.dstate, s.ngroups)
    ws = torch.empty(m3.block_workspace_size(dims), dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        m3.block_fwd(u, wts, out=out, workspace=ws)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        m3.block_fwd(u, wts, out=out, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    M, dm, H, P, N, G = s.batch * s.seqlen, s.d_model, s.nheads, s.headdim, s.dstate, s.ngroups
    HP, width = H * P, s.in_proj_width
    # per phase, the least time its own work allows: the two GEMMs at the bf16
    # peak or their operand bytes at HBM bandwidth, whichever is larger; the
    # prep, scan and gate kernels by the bytes they must move
    bw, pt = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops"] * 1e12
    # (the in_proj output is bf16: prep reads its B, C, dt and lam parts, the
    # scan reads x and the raw angles there, the gate reads z)
    t_in = max(2.0 * M * dm * width / pt, (M * dm * 2 + width * dm * 2 + M * width * 2) / bw)
    t_out = max(2.0 * M * HP * dm / pt, (M * HP * 2 + dm * HP * 2 + M * dm * 2) / bw)
    prep_b = M * ((2 * G * N + 2 * H) * 2 + 2 * G * N * 2 + 3 * H * 4)
    scan_b = M * (2 * HP * 2 + 3 * H * 4 + 2 * G * N * 2 + H * (N // 2) * 2)
    gate_b = M * HP * (2 + 2 + 2)
    t_lb = t_in + t_out + (prep_b + scan_b + gate_b) / bw
    return {"metric": "block Mtokens/s (fwd)", "value": M / (ms / 1e3) / 1e6, "unit": "Mtokens/s",
            "ms_per_step": ms, "steps": steps,
            "config": {"workload": s.name, "batch": s.batch, "seqlen": s.seqlen, "d_model": dm,
                       "nheads": H, "headdim": P, "dstate": N, "ngroups": G, "dtype": "bf16",
                       "weights": "random init"},
            "roofline": {"bound": "mixed", "t_lower_bound_ms": t_lb * 1e3,
                         "frac": t_lb * 1e3 / ms, "peak_hbm_gbs": peaks["hbm_gbs"],
                         "peak_bf16_tflops": peaks["bf16_tflops"], "peak_source": peaks["source"],
                         "gemm_tflop_per_step": 2.0 * M * (dm * width + HP * dm) / 1e12,
                         "note": "sum over phases of max(flops / bf16 peak, bytes / HBM) for the "
                                 "GEMMs and bytes / HBM for prep, scan (B, C per group, head bias applied inside) and gate"},
            "gpu_launches": 5 * steps,
            "note": "own kernels per call: in_proj GEMM, prep, scan, gate, out_proj GEMM"}


def bench_gemm(dev, peaks, steps: int = 10, warmup: int = 3):
    """The block's projection GEMM (m3ssd_gemm_bf16) alone at the model size's two
    shapes, against the measured bf16 peak; torch.matmul (cuBLAS) on the same
    operands is timed beside it for context."""
    import selective_state_space_m3ssd_b200 as m3
    from selective_state_space_m3ssd_b200.synth import BLOCKS
    s = BLOCKS["model"]
    M = s.batch * s.seqlen
    g = torch.Generator(device=dev).manual_seed(s.seed + 3)
    out = {}
    stream = torch.cuda.current_stream(dev)
    for name, (N, K) in (("in_proj", (s.in_proj_width, s.d_model)),
                         ("out_proj", (s.d_model, s.nheads * s.headdim))):
        A = torch.randn(M, K, device=dev, generator=g).bfloat16()
        W = (torch.randn(N, K, device=dev, generator=g) / K ** 0.5).bfloat16()
        D = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
        times = {}
        for impl, fn in (("own", lambda: m3.gemm_bf16(A, W, out=D)),
                         ("cublas", lambda: torch.matmul(A, W.t(), out=D))):
            for _ in range(warmup):
                fn()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            times[impl] = e0.elapsed_time(e1) / steps
        fl = 2.0 * M * N * K
        ach = fl / (times["own"] / 1e3) / 1e12
        out[name] = {"shape": [M, N, K], "ms": times["own"], "tflops": ach,
                     "frac": ach / peaks["bf16_tflops"],
                     "cublas_ms": times["cublas"],
                     "cublas_tflops": fl / (times["cublas"] / 1e3) / 1e12}
        del A, W, D
    tot_ms = out["in_proj"]["ms"] + out["out_proj"]["ms"]
    tot_fl = sum(2.0 * v["shape"][0] * v["shape"][1] * v["shape"][2] for v in out.values())
    ach = tot_fl / (tot_ms / 1e3) / 1e12
    return {"metric": "GEMM TFLOP/s (block projections)", "value": ach, "unit": "TFLOP/s",
            "ms_per_step": tot_ms, "steps": steps,
            "roofline": {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                         "peak_source": peaks["source"]},
            "shapes": out, "gpu_launches": 2 * steps}


def bench_backward(w, dev, steps, world, d, peaks):
    """The backward (m3ssd_bwd) on the forward's workload: dY, dhT synthetic,
    every gradient output written; inputs resident in HBM."""
    import selective_state_space_m3ssd_b200 as m3
    gen = torch.Generator().manual_seed(7)
    dY = torch.randn(tuple(d["X"].shape), generator=gen).to(d["X"].dtype).to(dev)
    dhT = torch.randn(w.batch, w.nheads, w.dstate, w.headdim, generator=gen).to(dev)
    args = [d[k] for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")]
    dims = m3.make_dims(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                        m3.BF16 if d["X"].dtype == torch.bfloat16 else m3.F32, 0)
    ws = torch.empty(m3.bwd_workspace_size(dims), dtype=torch.uint8, device=dev)
    grads = m3.bwd(*args, dY=dY, dhT=dhT, workspace=ws)  # warm-up, allocates the outputs
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        m3.bwd(*args, dY=dY, dhT=dhT, grads=grads, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    if world > 1:
        ms = max_over_ranks(ms, dev)
    algo = nbytes(*args, dY, dhT, *grads.values())
    flops = bwd_chunk_flops(w.batch, w.seqlen, w.nheads) * world
    executed = bwd_tc_mma_flops(w.batch, w.seqlen, w.nheads) * world
    tflops = flops / (ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    return {"metric": "bwd Mtokens/s", "value": w.batch * w.seqlen * world / (ms / 1e3) / 1e6,
            "unit": "Mtokens/s", "ms_per_step": ms, "steps": steps,
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak, "algo_flops_per_step": flops, "traffic": None,
                         "executed_mma_flops_per_step": executed,
                         "executed_frac": executed / (ms / 1e3) / 1e12 / peak,
                         "peak_source": peaks["source"] + " bf16 dense"},
            "hbm": {"algo_bytes_per_step": algo, "achieved_gbs": algo / (ms / 1e3) / 1e9,
                    "frac": algo / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]},
            "kernel": "bwd_tc_kernel + bwd_chunk_reduce_kernel (tcgen05 chunked backward, "
                      "2 launches)"}


def bwd_tc_mma_flops(b: int, L: int, H: int, N: int = 128, P: int = 64, Q: int = 64) -> int:
    """FLOPs the tensor-core backward's MMAs execute per call: every fp32
    operand split into two bf16 parts, three part products (four where they
    feed dtheta's suffix sums and dh_prev), X and dY exact; per chunk: G, Cbar
    h_prev and Bbar g at three parts (2 Q^2 N, 2 Q P N, 2 Q N P each), E and
    M^T dY at one and two (2 Q^2 P each), dh_prev, the two halves of dCbar and
    dBbar at four (2 N P Q, 2 Q N P and 2 Q^2 N), and the state pass at two."""
    per_chunk = 3 * (2 * Q * Q * N + 2 * Q * P * N + 2 * Q * N * P) + 2 * Q * Q * P * (1 + 2) + \
        4 * (2 * N * P * Q + 2 * 2 * Q * N * P + 2 * 2 * Q * Q * N) + 2 * (2 * N * P * Q)
    return b * H * -(-L // (Q - 1)) * per_chunk


def bwd_chunk_flops(b: int, L: int, H: int, N: int = 128, P: int = 64, Q: int = 64) -> int:
    """Product FLOPs of the chunked backward per call: per chunk of Q rows, the
    state pass's (W_end o Bbar)^T X (2 N P Q), then G = Cbar Bbar^T and
    E = dY X^T on their lower triangles (Q^2 N + Q^2 P), Bbar g (2 Q N P),
    M^T dY (Q^2 P), dY h^T (2 Q N P), WE Bbar and WE^T Cbar (2 Q^2 N),
    X g^T (2 Q N P) and Cbar^T (exp(cs) dY) (2 N P Q)."""
    per_chunk = 2 * N * P * Q + Q * Q * N + Q * Q * P + 2 * Q * N * P + Q * Q * P + \
        2 * Q * N * P + 2 * Q * Q * N + 2 * Q * N * P + 2 * N * P * Q
    return b * H * -(-L // (Q - 1)) * per_chunk


def fp32_simt_tflops(peaks: dict) -> float:
    """fp32 FMA peak of the SIMT pipes: 148 SMs x 128 lanes x 2 FLOP at the
    maximum SM clock (from the measured-peaks record, else 1,965 MHz)."""
    return 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    from selective_state_space_m3ssd_b200 import build as m3build
    if rank == 0 or world == 1:
        m3build.build()
    if world > 1:
        torch.distributed.barrier()
    peaks = load_peaks()
    w = rank_workload(WORKLOADS[FWD_KEY], rank)

    with ClockSampler(torch.cuda.get_device_properties(dev).index
                      if hasattr(torch.cuda.get_device_properties(dev), "index") else local) as clk:
        fw = bench_forward(w, dev, args.steps, args.warmup, world, rank)
        dec = bench_decode(dev, rank, max(1, args.decode_replays), peaks)
        mimo = bench_mimo_decode(dev, rank, peaks)
        blk = None if args.no_block else bench_block(dev, rank, peaks)
        gemm = None if args.no_block else bench_gemm(dev, peaks)
        bwd = None if args.no_backward else bench_backward(
            w, dev, max(1, min(args.steps, 3)), world, fw["dev_inputs"], peaks)
        others = {} if args.no_other_workloads else {
            k: forward_leg(k, dev, min(args.steps, 10), args.warmup, world, rank, peaks)
            for k in ("ssd", "long")}
        if not args.no_other_workloads:
            others["mimo"] = mimo_forward_leg(dev, min(args.steps, 10), args.warmup, world, rank,
                                              peaks)
            others["prefill"] = prefill_leg(dev, min(args.steps, 10), args.warmup, world, rank,
                                            peaks)
            others["sweep"] = chunk_sweep_leg(dev, min(args.steps, 5), args.warmup, world, rank,
                                              peaks)
    e2e = bench_e2e(w, dev, max(1, min(args.steps, 30)), 3, fw["inp"], world)

    tokens = w.batch * w.seqlen * args.steps * world
    value = tokens / (fw["ms_total"] / 1e3) / 1e6
    achieved = fw["algo_bytes"] / (fw["ms_per_step"] / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": fw["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(fwd_config(w), global_batch=w.batch * world,
                       parallelism=f"dp{world}" if world > 1 else "single"),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": recorded_traffic("fwd_chunk_siso", CHUNK_SRC),
                     "peak_source": peaks["source"], "algo_bytes_per_launch": fw["algo_bytes"],
                     "kernel": "fwd_chunk_kernel<theta, beta>"},
        "e2e": e2e,
        "gpu_launches": fw["launches"],
        "decode": dec,
        "mimo_decode": mimo,
        "block": blk,
        "gemm": gemm,
        "backward": bwd,
        "ssd_forward": others.get("ssd"),
        "long_forward": others.get("long"),
        "mimo_forward": others.get("mimo"),
        "prefill_forward": others.get("prefill"),
        "chunk_sweep": others.get("sweep"),
        "clocks": clk.summary(),
    }
    if world > 1:
        torch.distributed.barrier()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(fw["inp"])
    # a compact summary of every figure last, so that a tail of the line shows them
    line["summary"] = summary_of(line)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def summary_of(line: dict) -> dict:
    """Value, unit and roofline fraction of the headline and of each side figure."""
    def one(d):
        if not d:
            return None
        r = d.get("roofline") or {}
        return {"value": round(d["value"], 3), "unit": d["unit"],
                "ms_per_step": round(d["ms_per_step"], 4), "frac": round(r.get("frac", 0.0), 3)}
    out = {"forward_siso": one(line)}
    for k in ("ssd_forward", "long_forward", "mimo_forward", "prefill_forward", "chunk_sweep",
              "backward", "block", "gemm", "mimo_decode", "decode"):
        out[k] = one(line.get(k))
    sw = line.get("chunk_sweep")
    if sw:
        out["chunk_sweep"]["ms_by_chunk"] = {
            key: {q: round(v["ms_per_step"], 4) for q, v in rec["by_chunk"].items()}
            for key, rec in sw["sweep"].items()}
    return out


# ----------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ----------------------------------------------------------------------------

def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    w = WORKLOADS[FWD_KEY]
    inp = make_inputs(w)
    threads = oracle.default_threads()
    npairs = max(1, min(w.batch * w.nheads, threads))
    for _ in range(args.warmup):
        oracle_sample(inp, min(npairs, 2))
    total_th, total_s = 0, 0.0
    for _ in range(args.steps):
        th, dt, _ = oracle_sample(inp, npairs)
        total_th += th
        total_s += dt
    value = total_th / w.nheads / total_s / 1e6
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": dict(fwd_config(w), global_batch=w.batch, parallelism="host threads"),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"each step: {npairs} of {w.batch * w.nheads} (b,h) sequences, "
                                   f"full length L={w.seqlen}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile(args):
    """One kernel family alone, for ncu: the forward on the siso workload at
    L = 1024 (146 MB of inputs, above L2; a small case for full-section
    captures), the backward on one batch row at L = 1024 (a small case), the
    rank-4 MIMO decode step at batch 128 (134 MB of state, a small case), or
    the block at its model size (for launch lists only).  Prints
    one summary line; not a bench line."""
    import selective_state_space_m3ssd_b200 as m3
    from selective_state_space_m3ssd_b200 import build as m3build
    m3build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.profile in ("forward", "forward8"):
        # L = 1024 at batch 8 (146 MB of inputs, above L2; the same 256 sequences,
        # so the same single-walk launch as the benchmark's): a small case for
        # full-section captures; the full workload: the benchmark's own launch, for
        # one-pass counters
        w = WORKLOADS[FWD_KEY].with_(seqlen=1024) if args.profile == "forward" else WORKLOADS[FWD_KEY]
        fw = bench_forward(w, dev, args.steps, args.warmup, 1, 0)
        print(json.dumps({"profile": args.profile, "workload": w.name.replace(
                              "L4096", "L1024" if args.profile == "forward" else "L4096"),
                          "split": split_of(w, dev), "ms_per_step": fw["ms_per_step"],
                          "launches": fw["launches"]}))
    elif args.profile == "decode":
        # decode steps at half the decode batch: b128, fp32 cache (134 MB of
        # state, above L2), one step kernel and one b_prev update per call
        w = WORKLOADS["decode"].with_(batch=128, seqlen=args.warmup + args.steps)
        inp = make_inputs(w, device=dev)
        b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
        cache = m3.new_cache(b, H, P, N, G, dev)
        cache["ssm"].normal_(0, 0.3, generator=torch.Generator(device=dev).manual_seed(5))
        keys = ("X", "logdecay", "beta", "gamma", "B", "C", "theta")
        steps = {k: inp[k].transpose(0, 1).contiguous() for k in keys}
        y = torch.empty_like(steps["X"][0])
        for t in range(args.warmup + args.steps):
            m3.step(cache, *(steps[k][t] for k in keys), inp["D"], y_t=y)
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "decode", "workload": f"decode b{b} H{H} P{P} N{N} fp32 cache"}))
    elif args.profile == "backward":
        # one batch row of the forward's workload at L = 1024: 32 (b, h) CTAs of
        # the chunked backward
        w = WORKLOADS[FWD_KEY].with_(batch=1, seqlen=1024)
        inp = make_inputs(w)
        d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
        dY = torch.randn(tuple(d["X"].shape), generator=torch.Generator().manual_seed(7)).to(
            d["X"].dtype).to(dev)
        args_ = [d.get(k) for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D",
                                    "h0")]
        for _ in range(args.warmup + args.steps):
            m3.bwd(*args_, dY=dY)
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "backward", "workload": "siso shape b1 L1024 H32 P64 N128"}))
    elif args.profile == "wide":
        # the forward at chunk length 128 on the long workload's shape at a quarter of its
        # heads: b2 L32768 H12 (about 420 MB of inputs and outputs, above L2)
        w = WORKLOADS["long"].with_(nheads=12)
        d = make_inputs(w, device=dev)
        hT = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, dtype=torch.float32, device=dev)
        call = m3.PreparedFwd(*(d[k] for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta",
                                               "D", "h0")), hT=hT, chunk=128)
        for _ in range(args.warmup + args.steps):
            call()
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "wide", "workload": "long shape b2 L32768 H12, chunk 128"}))
    elif args.profile in ("long", "long12"):
        # the forward on the long workload (b2 L32768 H48: three segments a sequence),
        # or on its shape at a quarter of its heads (b2 L32768 H12, about 420 MB of
        # inputs and outputs, above L2: a small case of the segment pass)
        w = WORKLOADS["long"] if args.profile == "long" else WORKLOADS["long"].with_(nheads=12)
        d = make_inputs(w, device=dev)
        hT = torch.empty(w.batch, w.nheads, w.dstate, w.headdim, dtype=torch.float32, device=dev)
        call = m3.PreparedFwd(*(d[k] for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta",
                                               "D", "h0")), hT=hT)
        for _ in range(args.warmup + args.steps):
            call()
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": args.profile, "workload": f"long b{w.batch} L{w.seqlen} "
                          f"H{w.nheads}", "split": split_of(w, dev)}))
    elif args.profile == "prefill":
        # the fp32 prefill at a quarter of the decode batch: b64 L512 H32 (about 0.8 GB
        # of inputs and outputs, above L2), a small case of the fp32 chunked kernel
        w = WORKLOADS["decode"].with_(batch=64, seqlen=DECODE_PREFILL)
        fw = bench_forward(w, dev, args.steps, args.warmup, 1, 0)
        print(json.dumps({"profile": "prefill", "workload": f"decode prefill b{w.batch} "
                          f"L{w.seqlen} H{w.nheads} P{w.headdim} N{w.dstate} fp32",
                          "ms_per_step": fw["ms_per_step"]}))
    elif args.profile == "gemm":
        # the in_proj GEMM shape at a quarter of the block's tokens: 8192 x 6464 x 1024
        # (135 MB of operands and output, above L2), a small case for full captures
        from selective_state_space_m3ssd_b200.synth import BLOCKS
        s_ = BLOCKS["model"]
        M, N, K = 8192, s_.in_proj_width, s_.d_model
        g = torch.Generator(device=dev).manual_seed(11)
        A = torch.randn(M, K, device=dev, generator=g).bfloat16()
        W = (torch.randn(N, K, device=dev, generator=g) / K ** 0.5).bfloat16()
        D = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
        for _ in range(args.warmup + args.steps):
            m3.gemm_bf16(A, W, out=D)
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "gemm", "workload": f"in_proj GEMM {M} x {N} x {K} bf16"}))
    elif args.profile == "mimo_fwd":
        # the rank-4 MIMO prefill at batch 2 (about 290 MB of inputs and outputs,
        # above L2): a small case of the chunked MIMO kernel for full-section captures
        base, R = MIMO_WORKLOADS["mimo"]
        w = base.with_(batch=2)
        d = make_mimo_inputs(w, R, dev)
        Y = torch.empty_like(d["X"])
        args_ = [d[k] for k in ("X", "logdecay", "beta", "gamma", "B", "C", "theta", "D", "h0")]
        for _ in range(args.warmup + args.steps):
            m3.mimo_fwd(*args_, Y=Y)
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "mimo_fwd", "workload": w.name.replace("b8", "b2")}))
    elif args.profile == "mimo":
        # rank-4 MIMO decode steps at half the decode batch: b128, fp32 cache
        # (134 MB of state, above L2), one launch of the step kernel and one of
        # the b_prev update per call
        R = 4
        w = WORKLOADS["decode"].with_(batch=128)
        b, H, P, N, G = w.batch, w.nheads, w.headdim, w.dstate, w.ngroups
        gen = torch.Generator(device=dev).manual_seed(w.seed + 29)
        z = dict(device=dev, dtype=torch.float32)
        cache = m3.new_mimo_cache(b, H, P, N, G, R, dev)
        cache["ssm"].normal_(0, 0.3, generator=gen)
        x = torch.randn(b, H, P, R, generator=gen, **z)
        Bt = torch.randn(b, G, N, R, generator=gen, **z) / N ** 0.5
        Ct = torch.randn(b, G, N, R, generator=gen, **z) / N ** 0.5
        th = torch.randn(b, H, N // 2, generator=gen, **z) * 0.05
        ld = -torch.rand(b, H, generator=gen, **z) * 0.5
        be = torch.rand(b, H, generator=gen, **z) * 0.3
        ga = torch.rand(b, H, generator=gen, **z) * 0.5
        D = torch.randn(H, generator=gen, **z)
        y = torch.empty_like(x)
        for _ in range(args.warmup + args.steps):
            m3.mimo_step(cache, x, ld, be, ga, Bt, Ct, th, D, y_t=y)
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "mimo", "workload": f"mimo rank-{R} decode b{b} H{H} P{P} "
                          f"N{N} fp32 cache"}))
    else:
        from selective_state_space_m3ssd_b200.synth import BLOCKS, make_block
        s = BLOCKS["model"]
        u, wts = make_block(s, device=dev)
        out = torch.empty_like(u)
        for _ in range(args.warmup + args.steps):
            m3.block_fwd(u, wts, out=out)
        torch.cuda.synchronize(dev)
        print(json.dumps({"profile": "block", "workload": s.name}))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-replays", type=int, default=3,
                    help="replays of the 1000-step decode graph in the timed region")
    ap.add_argument("--no-block", action="store_true",
                    help="skip the Mamba-3 SISO block measurement")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward measurement")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the forward on the ssd and long workloads (side figures)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="omit the oracle timing (it never runs inside a GPU timed region)")
    ap.add_argument("--profile", choices=["forward", "forward8", "decode", "block", "backward",
                                          "mimo", "mimo_fwd", "gemm", "prefill", "wide", "long",
                                          "long12"],
                    help="run only a small case of one kernel family (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
