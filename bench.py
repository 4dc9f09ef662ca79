#!/usr/bin/env python
"""Benchmark of one routed-MoE layer forward pass (route -> permute -> [slot
cache step] -> grouped SwiGLU FFN -> combine) on B200, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W]          # headline + every workload (N = 1)
    python bench.py --config NAME [--T T] ...                    # one workload only
    python bench.py --impl reference ...                         # the CPU oracle on the host cores

One step = one layer pass over one batch of T tokens.  The headline is the
largest layer, the 753B-class NVFP4 layer at T = 16384; at N = 1 the line also
carries one record per other workload (35B decode T = 1/8/32/64, 35B prefill,
the 284B FP8 slot-cache trace, 753B NVFP4 decode), each timed the same way.
N > 1 (torchrun): every rank runs its own replica of the headline on its own
batch (tokens are independent, no data collective); value = all ranks' tokens
/ max-over-ranks time.  Prints one JSON line on rank 0.

Timing: W untimed warm-up steps, every CUDA graph captured, then exactly K
steps between CUDA events on the launching stream, synchronised on both sides
(barrier + max over ranks for N > 1).  Workloads whose expert bytes per step
are below 3x the L2 size rotate over that many copies of the slot pool, so
no step finds its weights in L2.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import expert_offloaded_edge_b200 as ftm  # noqa: E402
import synth  # noqa: E402

METRIC = "MoE-layer tokens/s; decode HBM GB/s & prefill TFLOP/s as % of B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
HEADLINE = ("753b_nvfp4", 16384)
SUITE = (("35b_decode", (1, 8, 32, 64)), ("35b_prefill", (8192,)), ("284b_trace", (32,)), ("753b_mxfp4", (16, 16384)),
         ("753b_nvfp4", (16,)))
K_BREAKDOWN = 40


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20, help="timed steps per workload")
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ftm", choices=["ftm", "reference"])
    p.add_argument("--config", default=None, choices=list(synth.CONFIGS),
                   help="run this workload only (default: the headline and, at N = 1, every workload)")
    p.add_argument("--T", type=int, default=None, help="tokens per step with --config (default: its largest)")
    p.add_argument("--experts", type=int, default=None,
                   help="with --config: the same layer with this many routed experts (and slots), e.g. a small "
                        "case of the same shape for a profiler capture")
    p.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying CUDA graphs")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=6.0, help="per CPU-baseline mode")
    p.add_argument("--bank-cache", default=os.path.join(tempfile.gettempdir(), "ftm_bench_banks"),
                   help="directory for packed expert banks reused across runs ('' = off)")
    return p.parse_args()


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 50):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", str(interval_ms)], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.p = None
        time.sleep(0.3)     # let the first sample land before the timed region starts

    def stop(self) -> dict:
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
        load = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- peaks / traffic
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


KERNEL_FILES = {"bf16": ("ftm_ffn.cu", "ftm_ffn_tc2.cu"), "f32": ("ftm_ffn.cu",), "fp8": ("ftm_ffn_fp8.cu",),
                "nvfp4": ("ftm_ffn_nvfp4.cu",), "mxfp4": ("ftm_ffn_nvfp4.cu",)}


def kernel_source_hash(wdtype: str) -> str:
    """Hash of the sources the dominant kernel of a dtype is built from."""
    h = hashlib.sha256()
    for n in KERNEL_FILES[wdtype] + ("ftm_gemm.cuh", "ftm_common.cuh"):
        with open(os.path.join(ROOT, "expert_offloaded_edge_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel: str, wdtype: str):
    """dram bytes per launch from the committed ncu summary (profiles/traffic.json),
    or None if absent or taken on a different version of the kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{workload}/{kernel}")
    if not e or e.get("source_hash") != kernel_source_hash(wdtype):
        return None
    return e.get("dram_bytes_per_launch")


def dtype_peak(pk: dict, src: str, wdtype: str):
    """Dense tensor peak of a dtype (TFLOP/s) and where it comes from: the measured
    sustained bf16 figure times the nominal dense ratio for fp8 (2) and fp4 (4)."""
    bf16 = float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))
    ratio = {"f32": 1.0, "bf16": 1.0, "fp8": 2.0, "nvfp4": 4.0, "mxfp4": 4.0}[wdtype]
    where = (f"bf16_tflops_sustained (of {src})" if ratio == 1.0 else
             f"derived: {ratio:g} x bf16_tflops_sustained (of {src}; nominal dense ratio)")
    return bf16 * ratio, where


# --------------------------------------------------------------------------- ranks
def job_throughput(local_ms: float, units_per_rank: int, dist, device) -> tuple:
    """Whole-job throughput of N independent replicas: the slowest rank's time
    (max over ranks) and all ranks' units divided by it.  dist=None: one rank."""
    world = 1
    ms = float(local_ms)
    if dist is not None:
        world = dist.get_world_size()
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms, units_per_rank * world / (ms / 1e3)


# --------------------------------------------------------------------------- layers
def source_hash() -> str:
    h = hashlib.sha256()
    for rel in ("synth/gen.c", "synth/__init__.py", "expert_offloaded_edge_b200/layout.py"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def packed_banks(cfg, cache_dir: str, local_rank: int, dist, seed: int = 0):
    """The layer's packed banks, drawn once and kept on the host's disk so later
    runs (and the other ranks of this one) read them instead of drawing again."""
    from synth.device import pack_banks
    if not cache_dir:
        return pack_banks(cfg, seed)
    tag = hashlib.sha1(repr(cfg).encode()).hexdigest()[:8]
    path = os.path.join(cache_dir, f"{cfg.name}_{source_hash()}_{tag}_s{seed}.npy")
    banks = None
    if local_rank == 0 and not os.path.exists(path):
        banks = pack_banks(cfg, seed)
        try:
            os.makedirs(cache_dir, exist_ok=True)
            tmp = path + f".tmp{os.getpid()}"
            with open(tmp, "wb") as f:
                np.save(f, banks)
            os.replace(tmp, path)
        except OSError:
            pass
    if dist is not None:
        dist.barrier()
    if banks is not None:
        return banks
    if os.path.exists(path):
        return np.load(path, mmap_mode="r")
    return pack_banks(cfg, seed)


def device_layer(cfg, args, local, dist, cache: bool = False):
    """The layer on this device.  cache: draw its banks once per host and keep
    them on disk (the headline layer, which every rank of a multi-GPU run and
    later runs on the same host stage again); the other layers are drawn here."""
    from synth.device import DeviceLayer
    return DeviceLayer(cfg, banks=packed_banks(cfg, args.bank_cache if cache else "", local, dist))


def workload_name(cfg, T):
    return f"{cfg.name} T={T}"


def workload_config(cfg, T, world):
    """The config block of a line: the same for this arm and the reference arm."""
    return {"workload": workload_name(cfg, T), "d": cfg.d, "E": cfg.E, "k": cfg.k, "I": cfg.I, "T": T,
            "has_shared": cfg.has_shared, "S": cfg.S, "wdtype": cfg.wdtype, "seed": 0,
            "parallelism": f"replicas x{world}"}


def routing_stats(dl, T, x):
    """Per-expert load of the benchmarked batch, from the library's own routing."""
    cfg = dl.cfg
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    gw = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    ftm.ftm_route(dl.desc, x, T, dl.w_router, dl.bias, ids, gw)
    torch.cuda.synchronize()
    return np.bincount(ids.cpu().numpy().ravel(), minlength=cfg.E)


def algorithmic(cfg, bl, T, counts):
    """Algorithmic bytes and flops of GEMM1 and of the whole layer step.  Bytes:
    the weight bytes of every expert touched (gate/up, down and their scales,
    i.e. its bank) plus the activations each GEMM reads and writes once."""
    wb = {"f32": 4, "bf16": 2, "fp8": 1, "nvfp4": 0.5, "mxfp4": 0.5}[cfg.wdtype]
    ab = 4 if cfg.act_dtype == "f32" else 2
    groups = int((counts > 0).sum()) + (1 if cfg.has_shared else 0)
    rows = T * cfg.k + (T if cfg.has_shared else 0)
    g1_w = 2 * cfg.I * cfg.d * wb + bl.s_gu_bytes + bl.s_t_bytes
    g2_w = cfg.d * cfg.I * wb + bl.s_d_bytes
    g1_bytes = groups * g1_w + rows * cfg.d * ab + rows * cfg.I * ab
    g2_bytes = groups * g2_w + rows * cfg.I * ab + rows * cfg.d * ab
    router_bytes = cfg.E * cfg.d * ab
    g1_flops = 2.0 * rows * cfg.d * 2 * cfg.I
    g2_flops = 2.0 * rows * cfg.I * cfg.d
    return {"groups": groups, "rows": rows, "gemm1_bytes": g1_bytes, "gemm2_bytes": g2_bytes,
            "layer_bytes": g1_bytes + g2_bytes + router_bytes + T * cfg.d * ab * 2,
            "weight_bytes": groups * (g1_w + g2_w), "gemm1_flops": g1_flops, "gemm2_flops": g2_flops,
            "layer_flops": g1_flops + g2_flops + 2.0 * T * cfg.E * cfg.d}


def rooflines(cfg, alg, g1_ms, step_ms, decode: bool):
    pk, src = peaks()
    if decode:
        peak = float(pk["hbm_gbs"])
        ach = alg["gemm1_bytes"] / (g1_ms * 1e-3) / 1e9
        lay = alg["layer_bytes"] / (step_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                "kernel": "gemm1 (grouped gate/up + SwiGLU)", "algorithmic_bytes": alg["gemm1_bytes"],
                "peak_source": f"hbm_gbs (of {src})",
                "layer": {"achieved": lay, "frac": lay / peak, "algorithmic_bytes": alg["layer_bytes"],
                          "what": "expert banks touched + router + activations, per step, over ms_per_step"}}
    peak, where = dtype_peak(pk, src, cfg.wdtype)
    ach = alg["gemm1_flops"] / (g1_ms * 1e-3) / 1e12
    lay = alg["layer_flops"] / (step_ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
            "kernel": "gemm1 (grouped gate/up + SwiGLU)", "algorithmic_flops": alg["gemm1_flops"],
            "peak_source": where,
            "layer": {"achieved": lay, "frac": lay / peak, "algorithmic_flops": alg["layer_flops"],
                      "what": "router + gate/up + down flops per step, over ms_per_step"}}


class Runner:
    """Graph-replayed (or eager) layer steps with per-kernel CUDA events.

    `kernels` are the kernel ids whose launches are bracketed by events; the
    timed region instruments only the dominant kernel (each event is one more
    graph node), a separate pass after it instruments all of them.  Steps
    rotate over `replicas` copies of the slot pool."""

    ALL = (ftm.binding.FTM_K_ROUTE, ftm.binding.FTM_K_PERMUTE, ftm.binding.FTM_K_GATHER,
           ftm.binding.FTM_K_GEMM1, ftm.binding.FTM_K_GEMM2, ftm.binding.FTM_K_COMBINE)

    def __init__(self, dl, T, x, use_graph: bool, replicas: int = 1, chunk: int = 20):
        from synth.device import Workspace
        self.dl, self.T = dl, T
        self.x = x
        self.out = torch.empty((T, dl.cfg.d), dtype=dl.out_dtype(), device="cuda")
        self.ws = Workspace(ftm.ftm_workspace_bytes(dl.desc, T))
        self.pools = [dl.pool] + [dl.pool.clone() for _ in range(replicas - 1)]
        bias = None if dl.bias is None else dl.bias.data_ptr()
        shared = None if dl.shared_bank is None else dl.shared_bank.data_ptr()
        self.weights = [ftm.LayerWeights(dl.w_router.data_ptr(), bias, p.data_ptr(), dl.slot_of_expert.data_ptr(),
                                         shared) for p in self.pools]
        self.use_graph = use_graph
        self.chunk = chunk
        self.graphs = {}
        self.stream = torch.cuda.Stream()
        self.kernels = (ftm.binding.FTM_K_GEMM1,)

    def step(self, i, x=None, out=None, stream=None):
        ftm.ftm_moe_layer_forward(self.dl.desc, self.weights[i % len(self.weights)], None,
                                  self.x if x is None else x, self.T, self.out if out is None else out,
                                  self.ws.ptr, self.ws.nbytes, self.stream if stream is None else stream)

    def launches_per_step(self) -> int:
        torch.cuda.synchronize()
        n0 = ftm.ftm_kernel_launches()
        self.step(0)
        n1 = ftm.ftm_kernel_launches()
        torch.cuda.synchronize()
        return n1 - n0

    def _events(self, n):
        evs = [{k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for k in self.kernels} for _ in range(n)]
        # torch creates the CUDA event on its first record(); the library re-records it later
        for ev in evs:
            for a, b in ev.values():
                a.record(self.stream)
                b.record(self.stream)
        self.stream.synchronize()
        return evs

    def _record_steps(self, evs):
        for i, ev in enumerate(evs):
            for k, (a, b) in ev.items():
                ftm.ftm_set_profile_events(k, a, b)
            self.step(i)
        for k in self.kernels:
            ftm.ftm_set_profile_events(k, None, None)

    def _plan(self, nsteps):
        out, done, tag = [], 0, 0
        while done < nsteps:
            n = min(self.chunk, nsteps - done)
            out.append((n, tag))
            tag ^= 1
            done += n
        return out

    def prepare(self, nsteps):
        """Capture every graph run(nsteps) replays (before any timed region)."""
        if not self.use_graph:
            return
        for n, tag in self._plan(nsteps):
            key = (n, tag, self.kernels)
            if key in self.graphs:
                continue
            evs = self._events(n)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(self.stream):
                self.step(0)          # one launch outside capture (sets kernel attributes)
                self.stream.synchronize()
                with torch.cuda.graph(g, stream=self.stream):
                    self._record_steps(evs)
            self.graphs[key] = (g, evs)
        torch.cuda.synchronize()

    def run(self, nsteps: int, collect: dict = None):
        """Enqueue nsteps steps on self.stream; per-kernel ms appended to collect."""
        if nsteps <= 0:
            return
        if not self.use_graph:
            evs = self._events(nsteps)
            with torch.cuda.stream(self.stream):
                self._record_steps(evs)
            if collect is not None:
                self.stream.synchronize()
                self._collect(evs, collect)
            return
        pending = []
        for n, tag in self._plan(nsteps):
            g, evs = self.graphs[(n, tag, self.kernels)]     # captured by prepare()
            if len(pending) == 2:     # the graph about to be replayed last ran two chunks ago
                pe = pending.pop(0)
                if collect is not None:
                    pe[-1][self.kernels[-1]][1].synchronize()
                    self._collect(pe, collect)
            g.replay()
            pending.append(evs)
        if collect is not None:
            for pe in pending:
                pe[-1][self.kernels[-1]][1].synchronize()
                self._collect(pe, collect)

    @staticmethod
    def _collect(evs, collect):
        for ev in evs:
            for k, (a, b) in ev.items():
                collect.setdefault(k, []).append(a.elapsed_time(b))


def e2e_pipelined(r: Runner, steps: int, dist):
    """End to end through the public call, every step: its tokens copied in from
    pinned host memory, the layer, its output copied back to pinned host
    memory.  Two buffer sets and separate copy streams let step i's copies run
    while step i +- 1 computes (PCIe is full duplex)."""
    T = r.T
    xs_h = [torch.empty_like(r.x, device="cpu").pin_memory() for _ in range(2)]
    for xh in xs_h:
        xh.copy_(r.x)
    outs_h = [torch.empty_like(r.out, device="cpu").pin_memory() for _ in range(2)]
    xs_d = [r.x, torch.empty_like(r.x)]
    outs_d = [r.out, torch.empty_like(r.out)]
    h2d, d2h, comp = torch.cuda.Stream(), torch.cuda.Stream(), r.stream
    ev_h = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_d = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            if i >= 2:
                h2d.wait_event(ev_c[b])           # step i-2 has read xs_d[b]
            with torch.cuda.stream(h2d):
                xs_d[b].copy_(xs_h[b], non_blocking=True)
            ev_h[b].record(h2d)
            comp.wait_event(ev_h[b])
            if i >= 2:
                comp.wait_event(ev_d[b])          # step i-2's output has left outs_d[b]
            r.step(i, x=xs_d[b], out=outs_d[b], stream=comp)
            ev_c[b].record(comp)
            d2h.wait_event(ev_c[b])
            with torch.cuda.stream(d2h):
                outs_h[b].copy_(outs_d[b], non_blocking=True)
            ev_d[b].record(d2h)

    run(3)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(h2d)
    run(steps)
    t1.record(d2h)
    torch.cuda.synchronize()
    ms, value = job_throughput(t0.elapsed_time(t1), steps * T, dist, "cuda")
    nb_in = r.x.numel() * r.x.element_size()
    nb_out = r.out.numel() * r.out.element_size()
    return {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": nb_in, "d2h_bytes_per_step": nb_out,
            "steps": steps, "ms_per_step": ms / steps,
            "launch": "eager ftm_moe_layer_forward; tokens in and outputs out through pinned host memory every "
                      "step, copies on their own streams overlapping the neighbouring steps' compute"}


def run_resident(dl, T, args, dist, local):
    """One resident-layer workload: warm-up, graphs captured, K timed steps, a
    per-kernel breakdown pass and the end-to-end pass."""
    cfg = dl.cfg
    K, W = args.steps, args.warmup
    x = dl.hidden(T)
    counts = routing_stats(dl, T, x)
    alg = algorithmic(cfg, dl.bl, T, counts)
    replicas = max(1, min(8, math.ceil(3 * L2_BYTES / max(1, alg["weight_bytes"]))))
    r = Runner(dl, T, x, not args.no_graph, replicas=replicas)
    per_step_launches = r.launches_per_step()
    with torch.cuda.stream(r.stream):
        for i in range(W):
            r.step(i)
    r.prepare(K)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    per_kernel = {}
    t0.record(r.stream)
    r.run(K, per_kernel)
    t1.record(r.stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    clk = clocks.stop()
    ms, value = job_throughput(ms, K * T, dist, "cuda")
    # per-kernel breakdown, after the timed region (every kernel bracketed by events)
    r.kernels = Runner.ALL
    r.prepare(K_BREAKDOWN)
    breakdown = {}
    r.run(K_BREAKDOWN, breakdown)
    torch.cuda.synchronize()
    e2e = e2e_pipelined(r, K, dist)
    status = ftm.ftm_device_status(True)
    kms = {ftm.KERNEL_NAMES[k]: float(np.mean(v)) for k, v in per_kernel.items()}
    kbreak = {ftm.KERNEL_NAMES[k]: float(np.mean(v)) for k, v in breakdown.items()}
    decode = alg["rows"] / max(1, alg["groups"]) < 64
    roof = rooflines(cfg, alg, kms.get("gemm1", float("nan")), ms / K, decode)
    roof["traffic"] = ncu_traffic(workload_name(cfg, T), "gemm1", cfg.wdtype)
    step_bytes = alg["weight_bytes"] * replicas
    rec = {
        "workload": workload_name(cfg, T), "value": value, "unit": "tokens/s", "ms_per_step": ms / K, "steps": K,
        "warmup": W, "dtype": cfg.wdtype, "config": workload_config(cfg, T, dist.get_world_size() if dist else 1),
        "l2": (f"inputs larger than L2: {alg['weight_bytes'] / 1e9:.3f} GB of expert banks per step"
               + (f", rotating over {replicas} copies of the slot pool ({step_bytes / 1e9:.2f} GB per cycle)"
                  if replicas > 1 else "")),
        "launch": "CUDA graph replay (graphs captured before the timed region)" if r.use_graph else "eager",
        "routing": {"active_experts": int((counts > 0).sum()), "rows": alg["rows"],
                    "max_rows_per_expert": int(counts.max()), "min_rows_active": int(counts[counts > 0].min())},
        "roofline": roof, "kernels_ms": kms, "kernels_ms_breakdown": kbreak, "e2e": e2e,
        "gpu_launches": per_step_launches * K, "launches_per_step": per_step_launches, "clocks": clk,
        "device_status": status,
    }
    if cfg.name == "35b_prefill":
        rec["routing"]["per_expert_rows"] = counts.tolist()
    return rec


def latency_floor(cfg, args, dist, local):
    """The same kernel chain as a T = 1 decode step of cfg, on a layer with
    d = I = 256 (about 3 MB of weights touched): the step time left when the
    bytes are negligible, i.e. the launch and dependency latency of the chain."""
    fcfg = synth.scaled(cfg, name=cfg.name + "_floor", d=256, I=256)
    dl = device_layer(fcfg, args, local, dist)
    rec = run_resident(dl, 1, args, dist, local)
    del dl
    return {"workload": f"latency floor: the {cfg.name} T=1 kernel chain at d = I = 256",
            "ms_per_step": rec["ms_per_step"], "steps": rec["steps"], "launch": rec["launch"],
            "launches_per_step": rec["launches_per_step"], "kernels_ms_breakdown": rec["kernels_ms_breakdown"],
            "clocks": rec["clocks"], "device_status": rec["device_status"]}


def run_trace(cfg, T, args, dist, local):
    """The decode trace over the LRU slot cache: one step = route, permute, cache
    update with miss copies (host sync), FFN, combine.  Warm-up = the first W
    steps of the trace, timed = the next K with the tokens resident in HBM,
    then end to end = the K steps after those, each step copying its tokens
    from pinned host memory and its output back (2K + W <= trace length)."""
    from synth.device import Workspace
    dl = device_layer(cfg, args, local, dist)
    W = min(args.warmup, cfg.trace_steps - 2)
    K = max(1, min(args.steps, (cfg.trace_steps - W) // 2))
    K2 = K
    xs = [dl.hidden(T, step=s) for s in range(W + K)]
    xs_host = [dl.hidden(T, step=s).cpu().pin_memory() for s in range(W + K, W + K + K2)]
    ws = Workspace(ftm.ftm_workspace_bytes(dl.desc, T))
    out = torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.Stream()
    copy_stream = torch.cuda.Stream()
    w = dl.weights()
    bl = dl.bl

    def step(s, evs=None):
        if evs:
            ftm.ftm_set_profile_events(ftm.binding.FTM_K_GEMM1, *evs)
        ftm.ftm_moe_layer_forward(dl.desc, w, dl.cache, xs[s], T, out, ws.ptr, ws.nbytes, stream, copy_stream)
        if evs:
            ftm.ftm_set_profile_events(ftm.binding.FTM_K_GEMM1, None, None)
        return dl.cache.last_hits, dl.cache.last_misses, dl.cache.last_distinct

    n0 = ftm.ftm_kernel_launches()
    for s in range(W):
        step(s)
    launches_warm = (ftm.ftm_kernel_launches() - n0) / max(1, W)
    torch.cuda.synchronize()
    evs = []
    for _ in range(K):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = ClockSampler(local)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hits = misses = distinct = 0
    n0 = ftm.ftm_kernel_launches()
    t0.record(stream)
    for i in range(K):
        h, m, dct = step(W + i, evs[i])
        hits, misses, distinct = hits + h, misses + m, distinct + dct
    t1.record(stream)
    torch.cuda.synchronize()
    launches = ftm.ftm_kernel_launches() - n0
    ms = t0.elapsed_time(t1)
    clk = clocks.stop()
    g1 = [a.elapsed_time(b) for a, b in evs]
    ms, value = job_throughput(ms, K * T, dist, "cuda")
    x_dev = torch.empty_like(xs[0])
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(K2):
        with torch.cuda.stream(stream):
            x_dev.copy_(xs_host[i], non_blocking=True)
        ftm.ftm_moe_layer_forward(dl.desc, w, dl.cache, x_dev, T, out, ws.ptr, ws.nbytes, stream, copy_stream)
        with torch.cuda.stream(stream):
            out_host.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, e2e_value = job_throughput(e0.elapsed_time(e1), K2 * T, dist, "cuda")
    status = ftm.ftm_device_status(True)
    pk, src = peaks()
    # The GEMM1 events bracket the launch of a step's hit experts and the shared
    # expert (the copied misses' launch follows the copies): its bytes are
    # (hits + 1) x gate/up bytes (+ scales), plus the activations of all rows (an
    # overcount of under 0.5%: the miss rows' activations go to the later launch)
    g1_w = 2 * cfg.I * cfg.d + bl.s_gu_bytes
    g2_w = cfg.d * cfg.I + bl.s_d_bytes
    groups = distinct / K + 1
    rows = T * cfg.k + T
    alg_g1 = (hits / K + 1) * g1_w + rows * (cfg.d + cfg.I) * 2
    layer_bytes = groups * (g1_w + g2_w) + rows * (cfg.d + cfg.I) * 4 + cfg.E * cfg.d * 2 + 2 * T * cfg.d * 2
    g1_ms = float(np.mean(g1))
    ach = alg_g1 / (g1_ms * 1e-3) / 1e9
    peak = float(pk["hbm_gbs"])
    return {
        "workload": workload_name(cfg, T) + f" trace steps {W}..{W + K - 1}", "value": value, "unit": "tokens/s",
        "ms_per_step": ms / K, "steps": K, "warmup": W, "dtype": cfg.wdtype,
        "config": workload_config(cfg, T, dist.get_world_size() if dist else 1),
        "l2": "inputs larger than L2: ~1.1 GB of FP8 expert banks touched per step",
        "launch": "eager (one host sync per step to read the miss list); the hit experts' FFN runs during the "
                  "miss copies, the copied misses' FFN after them",
        "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                     "kernel": "gemm1 (fp8 grouped gate/up + SwiGLU) of the hit experts and the shared expert, "
                               "which runs while the step's misses are copied", "algorithmic_bytes": alg_g1,
                     "peak_source": f"hbm_gbs (of {src})",
                     # the stored capture is of the single FFN launch a cache step made before
                     # the hit experts' launch was split from the misses': none for this one yet
                     "traffic": ncu_traffic(workload_name(cfg, T), "gemm1-hits", cfg.wdtype),
                     "layer": {"achieved": layer_bytes / (ms / K * 1e-3) / 1e9,
                               "frac": layer_bytes / (ms / K * 1e-3) / 1e9 / peak, "algorithmic_bytes": layer_bytes,
                               "what": "expert banks touched per step over the step time, which includes the "
                                       "PCIe miss copies the step waits for"}},
        "cache": {"hit_rate": hits / max(1, distinct), "misses_per_step": misses / K,
                  "h2d_gb_per_step": misses / K * bl.bank_bytes / 1e9,
                  "h2d_gbs_effective": misses * bl.bank_bytes / (ms * 1e-3) / 1e9},
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": int(xs_host[0].numel() * xs_host[0].element_size()),
                "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size()),
                "steps": K2, "trace_steps": f"{W + K}..{W + K + K2 - 1}",
                "launch": "eager; tokens copied in from pinned host memory and the output copied out every step, "
                          "on top of the miss copies the step already makes"},
        "gpu_launches": int(launches), "launches_per_step": launches / K, "launches_per_warmup_step": launches_warm,
        "clocks": clk, "device_status": status,
        "hybrid": run_trace_hybrid(dl, T, xs, W, K, stream, copy_stream, ms / K),
    }


def calibrate_bandwidths(dl, stream, reps: int = 5):
    """The two bandwidths of the miss split, measured the way the pages' `ft bench bw`
    calibration does: Bp = one expert bank copied from the pinned host pool to the
    device (CUDA events), Bh = one expert's FFN computed on the host for one row
    (wall clock), each as expert-bank bytes per second (GB/s)."""
    bb = int(dl.bl.bank_bytes)
    dst = torch.empty(bb, dtype=torch.uint8, device="cuda")
    src = dl.host_pool[:bb]
    with torch.cuda.stream(stream):
        for _ in range(2):
            dst.copy_(src, non_blocking=True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            dst.copy_(src, non_blocking=True)
        b.record(stream)
    torch.cuda.synchronize()
    bp = reps * bb / (a.elapsed_time(b) * 1e-3) / 1e9
    desc = dl.desc
    x = np.ascontiguousarray(dl.layer.hidden_storage(1, 0))
    y = np.zeros_like(x)
    nb = ftm.ftm_host_ffn_scratch_bytes(desc, 1)
    scratch = torch.empty(nb + 64, dtype=torch.uint8)
    sp = scratch.data_ptr() + (-scratch.data_ptr()) % 64
    bank = dl.host_pool.data_ptr()
    ftm.ftm_host_expert_ffn(desc, bank, x, 1, y, sp, nb, 0)
    t = []
    for _ in range(reps):
        t0 = time.perf_counter()
        ftm.ftm_host_expert_ffn(desc, bank, x, 1, y, sp, nb, 0)
        t.append(time.perf_counter() - t0)
    bh = bb / statistics.median(t) / 1e9
    return bp, bh


def run_trace_hybrid(dl, T, xs, W, K, stream, copy_stream, plain_ms):
    """The same trace steps through the bandwidth-adaptive miss split
    (ftm_moe_layer_forward_hybrid), from a cold cache like the offload run: W
    warm-up steps, then K timed with CUDA events on the layer's stream."""
    from synth.device import Workspace
    bp, bh = calibrate_bandwidths(dl, stream)
    for t in (dl.slot_of_expert, dl.expert_of_slot, dl.last_use):
        t.fill_(-1)
    dl.cache.step = 0
    torch.cuda.synchronize()
    ws = Workspace(ftm.ftm_hybrid_workspace_bytes(dl.desc, T))
    nb = ftm.ftm_hybrid_host_bytes(dl.desc, T)
    hbuf = torch.empty(nb, dtype=torch.uint8, pin_memory=True)
    h = ftm.Hybrid(bp, bh, 0, 0, 0, 0, 0.0, hbuf.data_ptr(), nb)
    out = torch.empty((T, dl.cfg.d), dtype=torch.bfloat16, device="cuda")
    w = dl.weights()

    def step(s):
        ftm.ftm_moe_layer_forward_hybrid(dl.desc, w, dl.cache, h, xs[s], T, out, ws.ptr, ws.nbytes, stream,
                                         copy_stream)
        return h.last_misses, h.last_host, h.last_host_ms

    for s in range(W):
        step(s)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    m = host = 0
    host_ms = 0.0
    t0.record(stream)
    for i in range(K):
        a, b, c = step(W + i)
        m, host, host_ms = m + a, host + b, host_ms + c
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / K
    return {"what": "the same trace steps with the bandwidth-adaptive miss split (q* policy): of each step's m "
                    "misses, q = round(m Bp / (Bp + Bh)) are copied over PCIe and computed on the GPU, m - q are "
                    "computed on the host CPU from the pinned host pool meanwhile; cold cache, as the offload run",
            "pcie_gbs": bp, "host_gbs": bh,
            "calibration": "Bp: one expert bank host->device, pinned (CUDA events); Bh: one expert's FFN for one "
                           "row on the host threads (wall clock); both in expert-bank bytes per second",
            "host_threads": os.cpu_count(), "steps": K, "warmup": W, "ms_per_step": ms,
            "ms_per_step_offload": plain_ms, "speedup_vs_offload": plain_ms / ms,
            "value": K * T / (ms * K * 1e-3), "unit": "tokens/s",
            "misses_per_step": m / K, "host_experts_per_step": host / K, "host_ffn_ms_per_step": host_ms / K,
            "device_status": ftm.ftm_device_status(True)}


def run_layers_pipeline(cfg, T, n_layers, args, local):
    """Prefill of n_layers layers of one shape (each with its own seed) through
    one slot cache of two layers' size (S = 2E), every layer's experts staged
    from pinned host memory: layer l+1's copies overlapped with layer l's
    compute, against staging then computing each layer.  One step = one pass
    over the stack, the output of layer l feeding layer l+1."""
    from synth.device import Workspace, to_device_storage
    E = cfg.E
    S = 2 * E
    desc = ftm.desc_for(synth.scaled(cfg, S=S))
    bl = ftm.ftm_get_bank_layout(desc)
    bb = bl.bank_bytes
    host_pool = torch.empty(n_layers * E * bb, dtype=torch.uint8, pin_memory=True)
    hp = host_pool.numpy()
    weights, keep = [], []
    for l in range(n_layers):
        banks = packed_banks(cfg, "", local, None, seed=l)
        hp[l * E * bb:(l + 1) * E * bb] = np.asarray(banks[:E]).reshape(-1)
        layer = synth.Layer(cfg, seed=l)
        wr = to_device_storage(layer.router_storage(), cfg.act_dtype)
        b = layer.bias()
        bias = None if b is None else torch.from_numpy(b).cuda()
        keep += [wr, bias]
        weights.append(ftm.LayerWeights(wr.data_ptr(), None if bias is None else bias.data_ptr(), None, None, None))
    pool = torch.zeros(S * bb, dtype=torch.uint8, device="cuda")
    soe = torch.full((n_layers * E,), -1, dtype=torch.int32, device="cuda")
    eos = torch.full((S,), -1, dtype=torch.int32, device="cuda")
    lu = torch.full((S,), -1, dtype=torch.int64, device="cuda")
    scratch = torch.zeros(ftm.ftm_slot_host_scratch_ints(desc), dtype=torch.int32, pin_memory=True)
    cache = ftm.SlotCache(soe.data_ptr(), eos.data_ptr(), lu.data_ptr(), 0, pool.data_ptr(), host_pool.data_ptr(),
                          scratch.data_ptr(), 0, 0, 0, 0, n_layers * E, 0)
    x0 = to_device_storage(synth.Layer(cfg, 0).hidden_storage(T), cfg.act_dtype)
    acts = [x0] + [torch.empty((T, cfg.d), dtype=torch.bfloat16, device="cuda") for _ in range(n_layers)]
    ws = Workspace(ftm.ftm_workspace_bytes(desc, T))
    stream, copy_stream = torch.cuda.Stream(), torch.cuda.Stream()
    passes = max(1, min(args.steps, 10))
    out = {}
    for mode in ("overlap", "serial"):
        used = None
        for _ in range(2):                            # warm-up passes
            used = ftm.ftm_moe_layers_forward(desc, weights, cache, acts[:-1], T, acts[1:], mode == "overlap",
                                              ws.ptr, ws.nbytes, stream, copy_stream)
        torch.cuda.synchronize()
        misses0 = 0
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(passes):
            ftm.ftm_moe_layers_forward(desc, weights, cache, acts[:-1], T, acts[1:], mode == "overlap", ws.ptr,
                                       ws.nbytes, stream, copy_stream)
            misses0 += cache.last_misses
        t1.record(stream)
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1)
        out[mode] = {"ms_per_pass": ms / passes, "ms_per_layer": ms / passes / n_layers, "overlap_ran": bool(used),
                     "last_layer_misses_per_pass": misses0 / passes,
                     # every layer misses like the last one: the cache holds two of the four layers
                     "h2d_gbs": misses0 * n_layers * bb / (ms * 1e-3) / 1e9 if misses0 else None}
    status = ftm.ftm_device_status(True)
    return {"workload": f"{cfg.name} x{n_layers} layers staged through one cache (S = 2E = {S}) T={T}",
            "value": T * n_layers / (out["overlap"]["ms_per_pass"] * 1e-3), "unit": "layer-tokens/s",
            "passes": passes, "overlap": out["overlap"], "serial": out["serial"],
            "speedup_overlap": out["serial"]["ms_per_pass"] / out["overlap"]["ms_per_pass"],
            "bank_bytes_per_layer": E * bb, "bound": "pcie (host-to-device expert copies)",
            "launch": "eager ftm_moe_layers_forward; layer l's output feeds layer l+1", "device_status": status}


# --------------------------------------------------------------------------- CPU oracle
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleTokens:
    """The oracle layer on one token at a time (router, its k experts, the shared
    expert, combine), on the first `ntok` tokens of the batch.  Their experts'
    weights are dequantised once, outside any timing: they are the layer's
    stored parameters."""

    def __init__(self, cfg, ntok: int = 2):
        import oracle
        self.oracle = oracle
        self.cfg = cfg
        self.layer = synth.Layer(cfg, 0, synth.load_redraws(cfg.name, max(cfg.T)) or {})
        self.x = self.layer.hidden_f32(ntok)
        self.Wr = self.layer.router_f32()
        self.b = self.layer.bias()
        ids, _, _ = oracle.route(self.x, self.Wr, self.b, cfg.k)
        want = set(ids.ravel().tolist()) | ({cfg.E} if cfg.has_shared else set())
        self.cache = {e: oracle.expert_weights_f32(self.layer, e) for e in sorted(want)}

    def token(self, t: int):
        o = self.oracle
        xs = self.x[t % len(self.x)][None, :]
        ids, g, _ = o.route(xs, self.Wr, self.b, self.cfg.k)
        o.moe_rows(self.layer, xs, [0], ids, g, weight_cache=self.cache)

    def timed(self, threads: int, seconds: float = None, per_thread: int = None):
        """Tokens processed by `threads` host threads (one oracle thread each), for
        `seconds` of wall time or `per_thread` tokens each; returns (tokens, s)."""
        done = [0] * threads

        def work(j):
            self.oracle.set_threads(1)
            n = 0
            while True:
                if per_thread is not None and n >= per_thread:
                    break
                if seconds is not None and time.perf_counter() - t0 >= seconds:
                    break
                self.token(j + n * threads)
                n += 1
            done[j] = n

        th = [threading.Thread(target=work, args=(j,)) for j in range(threads)]
        t0 = time.perf_counter()
        for t in th:
            t.start()
        for t in th:
            t.join()
        return sum(done), time.perf_counter() - t0


def cpu_baseline(cfg, T, seconds: float):
    ot = OracleTokens(cfg)
    ot.timed(1, per_thread=1)                     # warm
    n1, s1 = ot.timed(1, seconds=seconds)
    cores = host_cores()
    nc, sc = ot.timed(cores, seconds=seconds)
    return {"value": nc / sc, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "single_thread": {"value": n1 / s1, "unit": "tokens/s", "tokens": n1, "seconds": s1},
            "all_cores": {"value": nc / sc, "unit": "tokens/s", "tokens": nc, "seconds": sc, "threads": cores},
            "cpu_model": cpu_model(),
            "sample": (f"tokens 0..{len(ot.x) - 1} of the {workload_name(cfg, T)} batch, one token per oracle layer "
                       f"call (router, {cfg.k} experts{', shared expert' if cfg.has_shared else ''}, combine), "
                       f"{seconds:g} s on 1 thread, then {seconds:g} s on {cores} threads; expert weights "
                       f"dequantised beforehand")}


def reference_arm(args, rank, world):
    """The oracle as it stands, timed on the host cores on the same workload:
    each step = one token per host core, all cores at once."""
    if rank != 0:
        return
    name, T = (args.config, args.T or max(synth.CONFIGS[args.config].T)) if args.config else HEADLINE
    cfg = synth.CONFIGS[name]
    ot = OracleTokens(cfg)
    cores = host_cores()
    for _ in range(args.warmup):
        ot.timed(cores, per_thread=1)
    tot = 0.0
    for _ in range(args.steps):
        tot += ot.timed(cores, per_thread=1)[1]
    v = args.steps * cores / tot
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64-accumulate/f32",
            "data": "synthetic (seeded generator, weights N(0,0.02^2))",
            "config": workload_config(cfg, T, world),
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": f"each step = {cores} tokens of the {workload_name(cfg, T)} batch (tokens "
                                       f"0..{len(ot.x) - 1} in turn), one per host thread, each through the full "
                                       f"oracle layer (router, {cfg.k} experts"
                                       f"{', shared expert' if cfg.has_shared else ''}, combine)"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- main arm
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return reference_arm(args, rank, world)
    args.warmup = max(args.warmup, 3)
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    if args.config:
        head = (args.config, args.T or max(synth.CONFIGS[args.config].T))
        suite = ()
        if args.experts:
            c = synth.CONFIGS[args.config]
            synth.CONFIGS[args.config] = synth.scaled(c, E=args.experts, S=min(c.S, args.experts),
                                                      k=min(c.k, args.experts))
    else:
        head = HEADLINE
        suite = SUITE if world == 1 else ()
    records = []
    head_rec = None
    head_cfg = synth.CONFIGS[head[0]]
    for name, Ts in suite:
        cfg = synth.CONFIGS[name]
        if name == "35b_prefill":
            records.append(run_layers_pipeline(cfg, Ts[0], 4, args, local))
        if cfg.lru:
            for T in Ts:
                records.append(run_trace(cfg, T, args, dist, local))
            continue
        if name == "35b_decode":
            records.append(latency_floor(cfg, args, dist, local))
        dl = device_layer(cfg, args, local, dist, cache=name == head[0])
        for T in Ts:
            try:
                records.append(run_resident(dl, T, args, dist, local))
            except ftm.FtmError as e:     # a workload the library has no kernel for
                if e.status != ftm.binding.FTM_ERR_UNSUPPORTED:
                    raise
                records.append({"workload": workload_name(cfg, T), "unsupported": str(e)})
        if name == head[0]:
            head_rec = run_resident(dl, head[1], args, dist, local)
        del dl
        torch.cuda.empty_cache()
    if head_rec is None:
        if head_cfg.lru:
            head_rec = run_trace(head_cfg, head[1], args, dist, local)
        else:
            dl = device_layer(head_cfg, args, local, dist, cache=True)
            head_rec = run_resident(dl, head[1], args, dist, local)
            del dl
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_baseline(head_cfg, head[1], args.cpu_seconds)
        line = {
            "metric": METRIC, "value": head_rec["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": head_rec["steps"], "warmup": head_rec["warmup"], "ms_per_step": head_rec["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": head_rec["dtype"],
            "data": "synthetic (seeded generator, weights N(0,0.02^2), hidden N(0,1))",
            "config": dict(head_rec["config"], l2=head_rec["l2"], launch=head_rec["launch"]),
            "roofline": head_rec["roofline"],
            "cpu_baseline": cpu,
            "e2e": head_rec["e2e"],
            "gpu_launches": head_rec["gpu_launches"],
            "clocks": head_rec["clocks"],
            "routing": head_rec.get("routing"),
            "kernels_ms": head_rec.get("kernels_ms"),
            "kernels_ms_breakdown": head_rec.get("kernels_ms_breakdown"),
            "device_status": head_rec["device_status"],
            **{key: head_rec[key] for key in ("cache", "hybrid") if key in head_rec},
            "workloads": records,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
