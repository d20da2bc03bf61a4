"""Benchmark of the selective scan on B200: one JSON line on rank 0.

Default workload (the metric's shape): packed varlen bf16 scan, 16 sequences with lengths
drawn uniformly in [256, 4096], D = 2048 channels, N = 16 states, SiLU(z) gate.  A "step"
is one ssm_scan_fwd_varlen call over one packed batch (all steps of the hot path: staging,
softplus, discretisation, chunked scan, carry, contraction, gate, store, final states).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-secondary]

Multi-GPU (torchrun, one rank per GPU): every rank scans its own packed batch (seed offset by
rank), no collective on the data path ("scaling": "weak"); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "ncu_traffic.json")
SFU_PER_CLK_PER_SM = 16          # ex2/lg2/rcp results per clock per SM (measured on B200)
N_SM = 148
METRIC = "selective-scan tokens/s at D=2048,N=16; achieved HBM GB/s & roofline frac"
WORKLOAD = "varlen_bf16"


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("sm_max_mhz", 1965.0)), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1965.0, "fallback"


# The timed scan kernel (the chunked one, which the varlen workload takes) is defined by these
# sources and by the tile-shape line of its workload (the wide N=16 tile) in ssm_api.cu.
KERNEL_SOURCES = ("chunk_scan.cuh", "common.cuh")
KERNEL_SHAPE_MARKERS = ("template <> struct Shape<16, false>",)


def _code_only(text: str) -> str:
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash() -> str:
    """Hash of the timed scan kernel's code: its sources without comments and blank lines,
    plus its tile-shape line.  Comment edits and changes to other kernels or to host code
    keep the committed ncu counters valid; a change to the kernel's code or tile does not."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_15_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    with open(os.path.join(csrc, "ssm_api.cu"), encoding="utf-8") as f:
        shape = [ln.strip() for ln in f if any(m in ln for m in KERNEL_SHAPE_MARKERS)]
    h.update("\n".join(shape).encode())
    return h.hexdigest()[:16]


def ncu_traffic(key: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernels are unchanged."""
    try:
        with open(TRAFFIC_PATH) as f:
            t = json.load(f)
        e = t.get(key)
        if e and e.get("kernel_hash") == kernel_source_hash():
            return float(e["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        pass
    return None


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.6)
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------------------------ inputs

def rank_seed(rank: int) -> int:
    """Seed of a rank's packed batch: every rank scans its own batch (weak scaling)."""
    return workloads.CONFIGS[WORKLOAD]["seed"] + 1000 * rank


def reduce_over_ranks(dist, ms_local: float, tokens_local: float, device):
    """Job figures from per-rank ones: the slowest rank's time, the sum of all ranks' tokens."""
    import torch
    if dist is None:
        return ms_local, tokens_local
    t = torch.tensor([ms_local, float(tokens_local)], dtype=torch.float64, device=device)
    ms = t[0:1].clone()
    tok = t[1:2].clone()
    dist.all_reduce(ms, op=dist.ReduceOp.MAX)
    dist.all_reduce(tok, op=dist.ReduceOp.SUM)
    return float(ms[0]), float(tok[0])


def varlen_device_inputs(rank: int, device):
    import torch
    c = workloads.CONFIGS[WORKLOAD]
    seed = rank_seed(rank)
    lens = workloads.varlen_lengths(c["nseq"], c["len_lo"], c["len_hi"], seed)
    inp = workloads.varlen_inputs(lens, c["dim"], c["dstate"], c["dtype"], seed)
    T = inp.meta["total"]
    pitch = (T + 7) // 8 * 8           # rows padded to a 16-byte pitch

    def up(x, dt=torch.bfloat16):
        t = torch.zeros(x.shape[:-1] + (pitch,), dtype=dt)
        t[..., :T] = torch.from_numpy(x).to(dt)
        return t
    host = {k: up(getattr(inp, k)) for k in ("u", "delta", "z", "B", "C")}
    dev = {k: v.to(device) for k, v in host.items()}
    for k in ("A", "Dskip", "bias"):
        dev[k] = torch.from_numpy(getattr(inp, k)).to(device)
    dev["cu"] = torch.from_numpy(inp.cu_seqlens).to(device)
    host["cu"] = torch.from_numpy(inp.cu_seqlens)
    return inp, host, dev, T, pitch


def scan_counts(T, D, N, in_bytes, out_bytes, nseq):
    """Algorithmic bytes and exponentials of one scan launch."""
    bytes_ = T * D * (3 * in_bytes + out_bytes) + 2 * T * N * in_bytes + nseq * D * N * 4 + D * (N + 2) * 4
    exps = T * D * (N + 2)
    return bytes_, exps


# ------------------------------------------------------------------------------ CPU oracle

class CpuOracle:
    """The fp64 oracle on the host cores (all of them, or ``threads``) over a bounded channel
    sample of the packed batch.

    Channels are independent, so the sample's time scales to the full batch by D / channels."""

    def __init__(self, inp, budget_s: float, threads: int | None = None):
        import oracle
        oracle.build()
        self.oracle, self.inp = oracle, inp
        self.threads = threads or oracle.default_threads()
        self.D = inp.u.shape[0]
        self.T = inp.meta["total"]
        n0 = min(self.D, max(self.threads, 8))
        t_small = self._run(n0)
        self.nch = int(min(self.D, max(n0, n0 * budget_s / max(t_small, 1e-3))))

    def _run(self, nch):
        inp = self.inp
        ch = np.linspace(0, self.D - 1, nch).astype(np.int64)
        t0 = time.perf_counter()
        self.oracle.scan_varlen(inp.u[ch], inp.delta[ch], inp.B, inp.C, inp.A[ch], inp.cu_seqlens, inp.Dskip[ch],
                                inp.bias[ch], inp.z[ch], nthreads=self.threads)
        return time.perf_counter() - t0

    def measure(self):
        t = self._run(self.nch)
        return {"value": self.T * (self.nch / self.D) / t, "unit": "tokens/s", "cores": self.threads, "kind": "oracle",
                "sample": f"all {self.inp.meta['nseq']} sequences ({self.T} tokens) on {self.nch} of {self.D} "
                          f"channels, scaled by {self.D}/{self.nch}; {t:.2f} s wall"}


def cpu_oracle_rate(inp, budget_s: float = 12.0, single_budget_s: float = 6.0):
    """The oracle on all host cores, with the single-thread rate beside it."""
    out = CpuOracle(inp, budget_s).measure()
    one = CpuOracle(inp, single_budget_s, threads=1).measure()
    out["single_thread"] = {"value": one["value"], "unit": "tokens/s", "cores": 1, "sample": one["sample"]}
    return out


# ------------------------------------------------------------------------------ timing

def time_kernel(fn, steps, warmup, stream, flush=None):
    """Per-launch duration (ms) from CUDA events on the launching stream."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps
    total = 0.0
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    return total / steps


def long_run(name, steps, warmup, hbm_peak, sfu_peak, seqlen=None):
    """Kernel-only figures for one long single-sequence workload (inputs drawn on the device;
    `seqlen` shortens the sequence for profiler captures)."""
    import torch
    import selective_state_space_15_b200 as ssm
    stream = torch.cuda.current_stream()
    g = torch.Generator(device="cuda")
    c = workloads.CONFIGS[name]
    D, N, L = c["dim"], c["dstate"], seqlen or c["seqlen"]
    g.manual_seed(c["seed"])
    mk = lambda *s: torch.randn(*s, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)  # noqa: E731
    u, dl, z, B, C = mk(1, D, L), mk(1, D, L), mk(1, D, L), mk(1, N, L), mk(1, N, L)
    params = workloads.channel_params(np.random.default_rng(c["seed"]), D, N)
    A, Dsk, bias = (torch.from_numpy(x).cuda() for x in params)
    y = torch.empty_like(u)
    hl = torch.empty(1, D, N, device="cuda")
    ms = time_kernel(lambda: ssm.scan_fwd(u, dl, B, C, A, Dsk, bias, z, y=y, h_last=hl), steps, warmup, stream)
    nb, ne = scan_counts(L, D, N, 2, 2, 1)
    return {"ms": round(ms, 4), "tokens_per_s": L / (ms * 1e-3),
            "sfu_frac": round(ne / (ms * 1e-3) / sfu_peak, 4),
            "hbm_gbs": round(nb / (ms * 1e-3) / 1e9, 1), "hbm_frac": round(nb / (ms * 1e-3) / 1e9 / hbm_peak, 4)}


def decode_run(steps, warmup, hbm_peak):
    """Kernel-only figures for the decode workload: 256 of 1024 slots, D=5120, N=16."""
    import torch
    import selective_state_space_15_b200 as ssm
    stream = torch.cuda.current_stream()
    c = workloads.CONFIGS["decode_bf16"]
    prob = workloads.decode_problem(c["num_slots"], c["dim"], c["dstate"], c["R"], c["dtype"], c["seed"])
    pool = torch.from_numpy(prob.pool0).cuda()
    slots = torch.from_numpy(prob.slot_ids).cuda()
    A, Dsk, bias = (torch.from_numpy(x).cuda() for x in (prob.A, prob.Dskip, prob.bias))
    x = workloads.decode_step_inputs(prob, 0)
    bf = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)  # noqa: E731
    u, dl, z, B, C = bf(x["u"]), bf(x["delta"]), bf(x["z"]), bf(x["B"]), bf(x["C"])
    y = torch.empty_like(u)
    # the state (84 MB) fits in L2: read (not write) a 256 MB buffer between steps, so L2
    # ends up holding clean lines and no write-back of the flush lands inside the timed step.
    # The step is replayed from a CUDA graph: its kernel is shorter than a Python launch, and
    # the replay is queued while the flush runs, so the events bracket the kernel alone.
    scratch = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(3):
            ssm.state_update(pool, slots, u, dl, B, C, A, Dsk, bias, z, y=y)
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ssm.state_update(pool, slots, u, dl, B, C, A, Dsk, bias, z, y=y)
    ms = time_kernel(graph.replay, steps, warmup, stream, flush=lambda: scratch.sum())
    del graph
    R, D, N = c["R"], c["dim"], c["dstate"]
    nb = R * D * N * 4 * 2 + R * D * 2 * 4 + R * N * 2 * 2 + D * (N + 2) * 4
    return {"ms_per_step": round(ms, 5), "tokens_per_s": R / (ms * 1e-3),
            "hbm_gbs": round(nb / (ms * 1e-3) / 1e9, 1),
            "hbm_frac": round(nb / (ms * 1e-3) / 1e9 / hbm_peak, 4),
            "l2": "flushed (256 MB read) before each step", "launch": "CUDA graph replay"}


def small_batch_run(name, steps, warmup, sfu_peak, hbm_peak):
    """Kernel-only figures for the fixed-length float32 configs (seeded inputs uploaded once).
    The tiny one is launch-latency bound: its time is reported as the latency of one call."""
    import torch
    import selective_state_space_15_b200 as ssm
    stream = torch.cuda.current_stream()
    inp = workloads.config_inputs(name)
    up = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()  # noqa: E731
    u, dl, z, B, C, A, Dsk, bias = (up(getattr(inp, k)) for k in ("u", "delta", "z", "B", "C", "A", "Dskip", "bias"))
    y = torch.empty_like(u)
    b, D, L = u.shape
    N = A.shape[1]
    hl = torch.empty(b, D, N, device="cuda")
    scratch = torch.ones(64 << 20, device="cuda")      # 256 MB, read (not written) before each call
    ms = time_kernel(lambda: ssm.scan_fwd(u, dl, B, C, A, Dsk, bias, z, y=y, h_last=hl, stream=stream), steps, warmup,
                     stream, flush=lambda: scratch.sum())
    nb, ne = scan_counts(L * b, D, N, 4, 4, b)
    return {"us": round(ms * 1e3, 2), "tokens_per_s": b * L / (ms * 1e-3),
            "sfu_frac": round(ne / (ms * 1e-3) / sfu_peak, 4), "hbm_frac": round(nb / (ms * 1e-3) / 1e9 / hbm_peak, 4),
            "shape": f"batch {b}, D={D}, N={N}, L={L}, float32", "l2": "flushed (256 MB read) before each call",
            "launch": "one ssm_scan_fwd call through the binding (includes its workspace allocation)"}


def pool_prefill_run(steps, warmup, sfu_peak):
    """The varlen workload fed through ssm_scan_fwd_varlen_pool: 16 sequences whose states live
    in a 64-slot pool (read at the start, written back at the end of each sequence)."""
    import torch
    import selective_state_space_15_b200 as ssm
    stream = torch.cuda.current_stream()
    device = torch.device("cuda", torch.cuda.current_device())
    inp, _, dev, T, pitch = varlen_device_inputs(0, device)
    D, N, nseq = inp.u.shape[0], inp.A.shape[1], inp.meta["nseq"]
    pool = torch.zeros((64, D, N), dtype=torch.float32, device=device)
    slots = torch.arange(0, 4 * nseq, 4, dtype=torch.int32, device=device)
    y = torch.empty((D, pitch), dtype=torch.bfloat16, device=device)
    ms = time_kernel(lambda: ssm.scan_fwd_varlen_pool(dev["u"], dev["delta"], dev["B"], dev["C"], dev["A"], dev["cu"],
                                                      pool, slots, dev["Dskip"], dev["bias"], dev["z"], y=y, total=T,
                                                      stream=stream), steps, warmup, stream)
    _, ne = scan_counts(T, D, N, 2, 2, nseq)
    return {"ms": round(ms, 4), "tokens_per_s": T / (ms * 1e-3), "sfu_frac": round(ne / (ms * 1e-3) / sfu_peak, 4)}


def varlen_zoh_run(steps, warmup, sfu_peak):
    """The varlen workload with the zero-order-hold input matrix (ssm_scan_fwd_varlen, zoh)."""
    import torch
    import selective_state_space_15_b200 as ssm
    stream = torch.cuda.current_stream()
    device = torch.device("cuda", torch.cuda.current_device())
    inp, _, dev, T, pitch = varlen_device_inputs(0, device)
    D, N, nseq = inp.u.shape[0], inp.A.shape[1], inp.meta["nseq"]
    y = torch.empty((D, pitch), dtype=torch.bfloat16, device=device)
    hl = torch.empty((nseq, D, N), dtype=torch.float32, device=device)
    ms = time_kernel(lambda: ssm.scan_fwd_varlen(dev["u"], dev["delta"], dev["B"], dev["C"], dev["A"], dev["cu"],
                                                 dev["Dskip"], dev["bias"], dev["z"], y=y, h_last=hl, total=T,
                                                 stream=stream, zoh=True), steps, warmup, stream)
    _, ne = scan_counts(T, D, N, 2, 2, nseq)
    return {"ms": round(ms, 4), "tokens_per_s": T / (ms * 1e-3), "sfu_frac": round(ne / (ms * 1e-3) / sfu_peak, 4),
            "discretization": "zero-order hold"}


def decode_loop_run(hbm_peak, loop_steps=100):
    """A serving-style decode loop: `loop_steps` back-to-back decode steps (inputs cycling over 4
    token sets) captured in one CUDA graph; the active states (84 MB) stay in L2 between steps."""
    import torch
    import selective_state_space_15_b200 as ssm
    stream = torch.cuda.current_stream()
    c = workloads.CONFIGS["decode_bf16"]
    prob = workloads.decode_problem(c["num_slots"], c["dim"], c["dstate"], c["R"], c["dtype"], c["seed"])
    pool = torch.from_numpy(prob.pool0).cuda()
    slots = torch.from_numpy(prob.slot_ids).cuda()
    A, Dsk, bias = (torch.from_numpy(x).cuda() for x in (prob.A, prob.Dskip, prob.bias))
    bf = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)  # noqa: E731
    sets = []
    for k in range(4):
        x = workloads.decode_step_inputs(prob, k)
        sets.append([bf(x[n]) for n in ("u", "delta", "z", "B", "C")])
    ys = [torch.empty_like(sets[0][0]) for _ in range(4)]

    def loop():
        for i in range(loop_steps):
            u, dl, z, B, C = sets[i % 4]
            ssm.state_update(pool, slots, u, dl, B, C, A, Dsk, bias, z, y=ys[i % 4])
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        loop()
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        loop()
    ms = time_kernel(graph.replay, 5, 3, stream) / loop_steps
    del graph
    R, D, N = c["R"], c["dim"], c["dstate"]
    nb = R * D * N * 4 * 2 + R * D * 2 * 4 + R * N * 2 * 2 + D * (N + 2) * 4
    return {"ms_per_step": round(ms, 5), "tokens_per_s": R / (ms * 1e-3), "steps_per_graph": loop_steps,
            "hbm_gbs": round(nb / (ms * 1e-3) / 1e9, 1), "l2": "states resident in L2 between steps"}


def bwd_run(name, steps, warmup, sfu_peak):
    """Kernel figures of the backward (ssm_scan_bwd: segment pass, segment scan, reverse walk)
    on a fixed-length workload's shape (inputs and dy drawn on the device).  Its SFU count is
    twice the forward's D(N+2) per token (the forward exponentials are evaluated once in the
    segment pass and once more in the walk's recomputation)."""
    import torch
    import selective_state_space_15_b200 as ssm
    stream = torch.cuda.current_stream()
    c = workloads.CONFIGS[name]
    b, D, N, L = c["batch"], c["dim"], c["dstate"], c["seqlen"]
    dt = torch.float32 if c["dtype"] == "f32" else torch.bfloat16
    g = torch.Generator(device="cuda")
    g.manual_seed(c["seed"])
    mk = lambda *sh: torch.randn(*sh, generator=g, device="cuda", dtype=torch.float32).to(dt)  # noqa: E731
    u, dl, z, B, C, dy = mk(b, D, L), mk(b, D, L), mk(b, D, L), mk(b, N, L), mk(b, N, L), mk(b, D, L)
    A, Dsk, bias = (torch.from_numpy(x).cuda() for x in workloads.channel_params(np.random.default_rng(c["seed"]), D, N))
    ms = time_kernel(lambda: ssm.scan_bwd(u, dl, B, C, A, dy, Dsk, bias, z, stream=stream), steps, warmup, stream)
    ms_zoh = time_kernel(lambda: ssm.scan_bwd(u, dl, B, C, A, dy, Dsk, bias, z, stream=stream, zoh=True), steps,
                         warmup, stream)
    exps = 2 * b * L * D * (N + 2)
    return {"ms": round(ms, 4), "ms_zoh": round(ms_zoh, 4), "tokens_per_s": b * L / (ms * 1e-3),
            "sfu_frac": round(exps / (ms * 1e-3) / sfu_peak, 4),
            "shape": f"batch {b}, D={D}, N={N}, L={L}, {c['dtype']}", "exps_counted": "2 D (N+2) per token",
            "launches": "segment pass + segment scan + reverse walk (+ 6 memsets)"}


SSD_SHAPE = dict(batch=4, nheads=32, headdim=64, dstate=128, seqlen=4096, seed=910)


def ssd_run(steps, warmup, tensor_peak):
    """Kernel figures of the SSD chunked form on tcgen05 (ssm_ssd_fwd): 4 sequences x 32 heads x
    64 channels (D = 2048), N = 128, L = 4096, bf16; against the dense fp16/bf16 tensor peak."""
    import torch
    import selective_state_space_15_b200 as ssm
    stream = torch.cuda.current_stream()
    c = SSD_SHAPE
    inp = workloads.ssd_inputs(c["batch"], c["nheads"], c["headdim"], c["dstate"], c["seqlen"], seed=c["seed"])
    bf = lambda a: torch.from_numpy(a).cuda().to(torch.bfloat16)  # noqa: E731
    x, B, C = bf(inp.x), bf(inp.B), bf(inp.C)
    dt, A = torch.from_numpy(inp.dt).cuda(), torch.from_numpy(inp.A).cuda()
    y = torch.empty_like(x)
    hl = torch.empty(c["batch"], c["nheads"], c["headdim"], c["dstate"], device="cuda")
    ms = time_kernel(lambda: ssm.ssd_fwd(x, dt, A, B, C, y=y, h_last=hl, stream=stream), steps, warmup, stream)
    T, P, N = 128, c["headdim"], c["dstate"]
    chunks = c["batch"] * c["nheads"] * ((c["seqlen"] + T - 1) // T)
    flops = chunks * (2 * T * T * N + 3 * 2 * T * P * N)
    return {"ms": round(ms, 4), "tokens_per_s": c["batch"] * c["seqlen"] / (ms * 1e-3),
            "tflops": round(flops / (ms * 1e-3) / 1e12, 2), "tensor_frac": round(flops / (ms * 1e-3) / 1e12 / tensor_peak, 4),
            "shape": "4 sequences x 32 heads x 64 channels, N=128, L=4096, bf16 in/out, fp16 operands, fp32 accumulate",
            "flops_counted": "per head and 128-step chunk: 2 T T N + 6 T P N (C B^T, masked scores x V, C' H^T, state)"}


def secondary(steps, warmup, hbm_peak, sfu_peak):
    """Kernel-only figures for the small float32, long-sequence, pool-prefill and decode workloads (single GPU)."""
    out = {name: small_batch_run(name, steps, warmup, sfu_peak, hbm_peak) for name in ("tiny_f32", "batch_f32")}
    out.update({name: long_run(name, max(3, steps // 4), warmup, hbm_peak, sfu_peak)
                for name in ("long_bf16", "long_n128_bf16")})
    out["varlen_pool_bf16"] = pool_prefill_run(max(3, steps // 4), warmup, sfu_peak)
    out["varlen_zoh_bf16"] = varlen_zoh_run(max(3, steps // 4), warmup, sfu_peak)
    out["decode_bf16"] = decode_run(steps, warmup, hbm_peak)
    out["decode_loop_bf16"] = decode_loop_run(hbm_peak)
    out["bwd_batch_f32"] = bwd_run("batch_f32", max(3, steps // 8), warmup, sfu_peak)
    out["ssd_bf16"] = ssd_run(max(3, steps // 4), warmup, tensor_peak())
    return out


def tensor_peak():
    """Dense bf16 (= fp16) tensor peak, TFLOP/s: the measured burst figure, else the fallback."""
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        return 1590.0


# ------------------------------------------------------------------------------ arms

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    c = workloads.CONFIGS[WORKLOAD]
    lens = workloads.varlen_lengths(c["nseq"], c["len_lo"], c["len_hi"], c["seed"])
    inp = workloads.varlen_inputs(lens, c["dim"], c["dstate"], c["dtype"], c["seed"])
    # each step: the oracle over a channel sample sized so that the whole run takes ~2 minutes
    cpu = CpuOracle(inp, budget_s=min(10.0, max(0.05, 120.0 / max(1, args.steps + args.warmup))))
    per_step = []
    for i in range(args.warmup + args.steps):
        r = cpu.measure()
        if i >= args.warmup:
            per_step.append(r)
    value = statistics.median(r["value"] for r in per_step)
    T = inp.meta["total"]
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": T / value * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_desc(T)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": per_step[-1]["cores"], "kind": "oracle",
                             "sample": per_step[-1]["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def workload_desc(T):
    return (f"varlen_bf16: 16 packed sequences, lengths U[256,4096] ({T} tokens on rank 0), D=2048, N=16, "
            "bf16 in/out, fp32 state, SiLU(z) gate")


def run_ours(args, rank, world, local_rank):
    import torch
    import selective_state_space_15_b200 as ssm
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    ssm.load()
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    hbm_peak, sm_max, peak_kind = peaks()
    sfu_peak = N_SM * SFU_PER_CLK_PER_SM * sm_max * 1e6

    inp, host, dev, T, pitch = varlen_device_inputs(rank, device)
    D, N, nseq = inp.u.shape[0], inp.A.shape[1], inp.meta["nseq"]
    y = torch.empty((D, pitch), dtype=torch.bfloat16, device=device)
    hl = torch.empty((nseq, D, N), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step():
        ssm.scan_fwd_varlen(dev["u"], dev["delta"], dev["B"], dev["C"], dev["A"], dev["cu"], dev["Dskip"],
                            dev["bias"], dev["z"], y=y, h_last=hl, total=T, stream=stream)

    # ---- kernel-resident timing (inputs in HBM; 0.58 GB of inputs per step > 126 MB L2)
    sampler = ClockSampler(local_rank) if rank == 0 else None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_local = e0.elapsed_time(e1)
    if dist:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    tokens_local = T * args.steps
    ms_max, tokens_all = reduce_over_ranks(dist, ms_local, tokens_local, device)
    value = tokens_all / (ms_max * 1e-3)
    ms_per_step = ms_max / args.steps

    if args.kernel_only:
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                              "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                              "mode": "kernel-only (ncu capture; e2e, CPU and secondary legs not run)"}))
        return 0

    # ---- end to end through the public API with host buffers (pinned), copies timed.
    # Steps are pipelined over three streams and two sets of device buffers: the host->device
    # copy of step k+1 and the device->host copy of step k-1 overlap the scan of step k
    # (PCIe moves both directions at once), as a serving loop would run it.
    pinned = {k: v.pin_memory() for k, v in host.items()}
    y_hosts = [torch.empty((D, pitch), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hl_hosts = [torch.empty((nseq, D, N), dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = y_hosts[0].numel() * y_hosts[0].element_size() + hl_hosts[0].numel() * hl_hosts[0].element_size()
    devs = [dev, {k: torch.empty_like(v) for k, v in dev.items()}]
    for k in ("A", "Dskip", "bias"):
        devs[1][k] = dev[k]
    ys = [y, torch.empty_like(y)]
    hls = [hl, torch.empty_like(hl)]
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("loaded", "computed", "stored")}
    for b in range(2):  # every buffer starts free
        for n in ("computed", "stored"):
            ev[n][b].record(stream)

    def e2e_step(i):
        b = i % 2
        d = devs[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev["computed"][b])          # the scan of step i-2 has read buffer b
            for k, v in pinned.items():
                d[k].copy_(v, non_blocking=True)
            ev["loaded"][b].record(s_in)
        stream.wait_event(ev["loaded"][b])
        stream.wait_event(ev["stored"][b])              # y/h_last of step i-2 have been copied out
        ssm.scan_fwd_varlen(d["u"], d["delta"], d["B"], d["C"], d["A"], d["cu"], d["Dskip"], d["bias"], d["z"],
                            y=ys[b], h_last=hls[b], total=T, stream=stream)
        ev["computed"][b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["computed"][b])
            y_hosts[b].copy_(ys[b], non_blocking=True)
            hl_hosts[b].copy_(hls[b], non_blocking=True)
            ev["stored"][b].record(s_out)
    e2e_steps = max(3, min(args.steps, 20))
    for i in range(min(args.warmup, 3)):
        e2e_step(i)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    s_in.wait_stream(s_out)
    s_in.wait_stream(stream)
    f1.record(s_in)
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1)
    e2e_tokens = T * e2e_steps
    e2e_ms, e2e_tokens = reduce_over_ranks(dist, e2e_ms, e2e_tokens, device)
    e2e_value = e2e_tokens / (e2e_ms * 1e-3)

    extra = None
    if rank == 0 and world == 1 and not args.no_secondary:
        extra = secondary(args.steps, args.warmup, hbm_peak, sfu_peak)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    # roofline of the (single) kernel on rank 0's batch, per launch
    launch_s = ms_local / args.steps * 1e-3
    nbytes, nexps = scan_counts(T, D, N, 2, 2, nseq)
    traffic = ncu_traffic(WORKLOAD)
    cpu = cpu_oracle_rate(inp) if world == 1 else None
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(T), "tokens_per_step_rank0": T,
                   "global_batch_tokens": tokens_all / args.steps,
                   "l2": "inputs 0.58 GB per step > 126 MB L2; no flush",
                   "parallelism": f"dp{world} (independent batches)"},
        "roofline": {"bound": "alu", "unit": "Gexp/s", "achieved": nexps / launch_s / 1e9, "peak": sfu_peak / 1e9,
                     "frac": nexps / launch_s / sfu_peak, "traffic": traffic,
                     "peak_note": f"MUFU: {N_SM} SMs x {SFU_PER_CLK_PER_SM} results/clk (15.96 measured, "
                                  f"profiles/mufu_rate_b200.md) x {sm_max:.0f} MHz; counted: D(N+2) exponentials "
                                  "per token (N exp(Delta A), one in softplus, one in the gate) -- the algorithm's "
                                  "lower bound",
                     "mufu_ops_per_token_kernel": D * (N + 3),
                     "mufu_note": "the timed (chunked) kernel issues D(N+3) MUFU operations per token: the N "
                                  "exponentials, one ex2 per 16-step lane segment and state for the segment "
                                  "product (D N / 16), one in softplus, one tanh in the gate"},
        "roofline_hbm": {"bound": "hbm", "unit": "GB/s", "achieved": nbytes / launch_s / 1e9, "peak": hbm_peak,
                         "frac": nbytes / launch_s / 1e9 / hbm_peak, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": nbytes},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "pipeline": "H2D of step k+1 and D2H of step k-1 overlap the scan of step k"},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if extra:
        line["secondary"] = extra
    print(json.dumps(line))
    return 0


def run_other(args, rank, world, local_rank):
    """--kernel-only --workload X: the kernel of a secondary workload alone, on one GPU."""
    import torch
    import selective_state_space_15_b200 as ssm
    if rank != 0:
        return 0
    torch.cuda.set_device(local_rank)
    ssm.load()
    hbm_peak, sm_max, _ = peaks()
    sfu_peak = N_SM * SFU_PER_CLK_PER_SM * sm_max * 1e6
    if args.workload == "decode_bf16":
        r = decode_run(args.steps, args.warmup, hbm_peak)
    elif args.workload == "bwd_batch_f32":
        r = bwd_run("batch_f32", args.steps, args.warmup, sfu_peak)
    elif args.workload == "ssd_bf16":
        r = ssd_run(args.steps, args.warmup, tensor_peak())
    elif args.workload in ("tiny_f32", "batch_f32"):
        r = small_batch_run(args.workload, args.steps, args.warmup, sfu_peak, hbm_peak)
    else:
        r = long_run(args.workload, args.steps, args.warmup, hbm_peak, sfu_peak, args.seqlen)
    print(json.dumps({"workload": args.workload, "seqlen": args.seqlen, "steps": args.steps, "warmup": args.warmup, **r,
                      "mode": "kernel-only (ncu capture)"}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-secondary", action="store_true", help="skip the long-sequence/decode figures")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[WORKLOAD, "long_bf16", "long_n128_bf16", "decode_bf16", "tiny_f32", "batch_f32",
                             "bwd_batch_f32", "ssd_bf16"],
                    help="with --kernel-only: time another workload's kernel alone (for ncu captures)")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="with --kernel-only and a long workload: a shorter sequence (profiler captures)")
    ap.add_argument("--kernel-only", action="store_true",
                    help="only the warm-up and timed kernel steps (for ncu captures); prints a short line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload != WORKLOAD and not args.kernel_only:
        ap.error("--workload other than the metric's needs --kernel-only")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.workload != WORKLOAD:
        return run_other(args, rank, world, local_rank)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
