#!/usr/bin/env python
"""Benchmark of the FMDQ differential linear hot path on B200.

One step = one pass of the whole hot path over one batch: for every layer of
the workload, the quantizer (K1) and the slice GEMM with its fused epilogue
(K2), through the C ABI.  Headline workload: the Latte-like video DiT FFN,
batch 4 x 16 frames x 256 tokens = 16384 tokens, 1152 -> 4608 -> 1152, bf16
activations, int8 weights (the largest of the five workloads; it fits one
GPU).  On one GPU the same line also carries the DiT-XL/2 256px FFN pair, the
PixArt 1024px layer and the 28-layer x 50-step timestep sweep with its forced
all-2-bit and all-8-bit runs (`per_config`, `sweep`).

Metric: dense-equivalent int8 TOPS, sum over layers of 2*M*N*K per step / step
time, with the quantizer's HBM GB/s and the slice GEMM's tensor throughput as
fractions of the measured peaks.  Inputs live in HBM and rotate over buffer
sets larger than L2, so no timed step reuses L2-resident data.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 it is launched with torch.distributed.run; every rank runs its own
batch (weak scaling, no data-path collective); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FMDQ linear dense-equiv TOPS & % int8 tensor peak; quantizer GB/s vs HBM"
INT8_PER_BF16 = 2.0  # nominal dense int8 : bf16 tensor throughput on B200 (4.5 : 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HEADLINE_CONFIG = 4


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=HEADLINE_CONFIG,
                    help="headline workload (4: Latte video FFN; 2: DiT-XL/2 FFN pair; 3: PixArt layer)")
    ap.add_argument("--extra-configs", default="2,3",
                    help="further workloads measured on one GPU and reported under per_config ('' for none)")
    ap.add_argument("--extra-steps", type=int, default=1200, help="timed steps of each extra workload")
    ap.add_argument("--sweep-steps", type=int, default=50,
                    help="steps of the 28-layer timestep sweep on one GPU (0 to skip)")
    ap.add_argument("--extreme-reps", type=int, default=5, help="timed steps of each forced-width sweep run")
    ap.add_argument("--sets", type=int, default=3, help="rotating input sets (together larger than L2)")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--xprev", choices=["swap", "copy"], default="copy",
                    help="swap: X_t and X_{t-1} stay resident and trade buffers each step (no refresh copy); "
                         "copy: the quantizer copies X_t into one x_prev cache")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", action="store_true",
                    help="skip the chained FFN pair, the dynamic base and the sparse attention runs")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--mode", choices=["graph", "eager"], default="graph",
                    help="graph: each step replays a captured CUDA graph; eager: C-ABI calls per step")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- peaks

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# the sources that decide the benchmarked step's kernels and their launches
STEP_SOURCES = ("fmdq_device.cuh", "fmdq_gemm.cu", "fmdq_host.cu", "fmdq_internal.h", "fmdq_quant.cu")


def kernel_source_sha():
    """Hash of the step's kernel sources without their comments (a comment
    edit does not make recorded counters stale; any code change does)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "differential_quantized_gemm_b200", "csrc")
    for f in STEP_SOURCES:
        text = open(os.path.join(csrc, f), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(f.encode())
        h.update("\n".join(line.rstrip() for line in text.splitlines() if line.strip()).encode())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else {})."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return {}
    out, sha = {}, None
    for line in open(p):
        line = line.strip()
        if line.startswith("source_sha="):
            sha = line.split("=", 1)[1]
        elif line and not line.startswith("#") and "=" in line:
            k, v = line.split("=", 1)
            try:
                out[k] = float(v)
            except ValueError:
                pass
    return out if sha == kernel_source_sha() else {}


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# -------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str, enabled: bool = True):
        self.proc = None
        self.lines = []
        if not enabled:
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self, t0: float, t1: float):
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(f[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                rows.append((ts, float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 - 1 <= r[0] <= t1 + 1] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r[1] for r in inside if r[1] > 0.5 * r[2]] or [r[1] for r in inside]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ------------------------------------------------------------ workload

class Layer:
    """Device buffers and prebuilt C-ABI arguments of one layer in one input set."""

    def __init__(self, inp, torch, nat, swap):
        spec = inp.spec
        self.swap = swap
        self.spec = spec
        dev = "cuda"

        def bf(a):
            return torch.from_numpy(a).view(torch.bfloat16).to(dev) if spec.dtype == "bf16" else \
                torch.from_numpy(a).to(dev)

        self.x_a = bf(inp.x_t)           # X at even uses
        self.x_b = bf(inp.x_prev)        # X at odd uses
        self.x_prev = None if swap else self.x_b.clone()  # cache (copy mode)
        self.y_prev = bf(inp.y_prev)     # cache, updated in place
        self.w_q = torch.from_numpy(inp.w_q).to(dev)
        self.w_scale = torch.from_numpy(inp.w_scale).to(dev)
        self.ws = nat.Workspace(spec.M, spec.K)
        self.base = 2.0 ** spec.lb
        self.cfg = nat.TileCfg(16, spec.t0, spec.force_bits, nat.FLAG_NO_XPREV_REFRESH if swap else 0,
                               ctypes.c_void_p(self.ws.ptr), self.ws.nbytes, None, None)
        self.m_x = [nat.mat(self.x_a), nat.mat(self.x_b)]
        self.m_xp = None if swap else nat.mat(self.x_prev)
        self.m_y = nat.mat(self.y_prev)
        self.m_w = nat.mat(self.w_q)
        self.ws_ptr = ctypes.c_void_p(self.w_scale.data_ptr())

    def tensors(self):
        return [t for t in (self.x_a, self.x_b, self.x_prev, self.y_prev, self.w_q, self.w_scale, self.ws.buf)
                if t is not None]

    def xp(self, parity):
        """X_{t-1}: the other buffer (swap), or the cache (copy)."""
        return self.m_x[1 - parity] if self.swap else self.m_xp

    def quantize(self, L, parity, stream):
        return L.dstar_fmdq_quantize(ctypes.byref(self.m_x[parity]), ctypes.byref(self.xp(parity)), self.base,
                                     ctypes.byref(self.cfg), stream)

    def gemm(self, L, stream):
        return L.dstar_fmdq_slice_gemm(ctypes.byref(self.m_w), self.ws_ptr, ctypes.byref(self.m_y), self.base,
                                       ctypes.byref(self.cfg), ctypes.byref(self.m_y), stream)

    def linear(self, L, parity, stream):
        return L.dstar_fmdq_linear(ctypes.byref(self.m_x[parity]), ctypes.byref(self.xp(parity)), ctypes.byref(self.m_y),
                                   ctypes.byref(self.m_w), self.ws_ptr, self.base, ctypes.byref(self.cfg),
                                   ctypes.byref(self.m_y), stream)


def max_over_ranks(value: float, device="cpu") -> float:
    """The largest of every rank's value (the job's time is its slowest rank's);
    the value itself in a single-process run."""
    import torch
    import torch.distributed as td
    if not (td.is_available() and td.is_initialized()) or td.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def job_tops(world: int, ops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank does the same work per step (weak
    scaling), and the step takes the slowest rank's time."""
    return world * ops_per_rank / (ms_per_step * 1e-3) / 1e12


XPREV_DESC = {
    "swap": "X_t and X_{t-1} resident in two buffers that trade roles each step (DSTAR_FLAG_NO_XPREV_REFRESH)",
    "copy": "one x_prev cache per layer, refreshed with X_t by the quantizer",
}


def workload_config(cfg, inputs, world, xprev="copy"):
    """The `config` of the JSON line: the workload, the same for both arms."""
    from differential_quantized_gemm_b200 import synth
    return {"workload": synth.CONFIG_NAMES[cfg],
            "layers": [f"{i.spec.name} M={i.spec.M} K={i.spec.K} N={i.spec.N}" for i in inputs],
            "base_scale": f"2^{inputs[0].spec.lb}", "tile_tokens": 16,
            "x_prev": XPREV_DESC[xprev],
            "parallelism": f"{world} replica(s), one batch per GPU, no collective"}


def workload_inputs(cfg, rank):
    from differential_quantized_gemm_b200 import synth
    seed = None if rank == 0 else cfg + 7919 * rank
    return [synth.make_layer(cfg, li, seed=seed) for li in range(len(synth.config_layers(cfg)))]


def algorithmic_k1_bytes(spec, ws_sections, in_bytes=2, refresh=True):
    """Bytes K1 must move for one launch: read X_t and X_{t-1}, write X_t into
    the cache (only when it refreshes one), write plane 0 (and plane 1 for
    two-plane tiles), the encoded stream (8 bytes per slice record) and the
    per-sub-channel FPoT and width."""
    import numpy as np
    M, K = spec.M, spec.K
    count = ws_sections["count"].cpu().numpy().astype(np.int64)
    planes = ws_sections["planes"].cpu().numpy()
    rows2 = int((planes == 2).sum()) * 16
    return ((3 if refresh else 2) * M * K * in_bytes + M * K + rows2 * K + int(count.sum()) * 8 + 2 * (M // 16) * K)


def algorithmic_k2(spec, ws_sections, out_bytes=2):
    """Ops (dense-equivalent 2MNK and issued incl. plane 1) and bytes of one
    slice-GEMM launch: read Y_{t-1}, write Y_t, read W and the operand planes."""
    import numpy as np
    M, K, N = spec.M, spec.K, spec.N
    mask = ws_sections["mask1"].cpu().numpy().view(np.uint32)
    planes = ws_sections["planes"].cpu().numpy()
    T = M // 16
    nb = (M + 127) // 128
    chunks1 = 0
    for b in range(nb):
        m = np.bitwise_or.reduce(mask[b * 8:min(T, b * 8 + 8)], axis=0)
        chunks1 += sum(bin(int(x)).count("1") for x in np.atleast_1d(m))
    dense_ops = 2.0 * M * N * K
    issued = dense_ops + 2.0 * 128 * N * 128 * chunks1
    bytes_ = 2 * M * N * out_bytes + N * K + M * K + chunks1 * 128 * 128
    return dense_ops, issued, bytes_, int((planes > 2).sum())


def kernel_rows(inputs, stats, k1_ms, k2_ms, peaks, spread=None):
    """Per launch: time, achieved rate and fraction of the bound that applies
    (HBM for the quantizer; for the slice GEMM the larger of tensor and HBM
    time at the measured peaks); with spread ({(kernel, layer index): (median,
    min, max) ms}) also the spread of the sampled launches."""
    hbm = peaks["hbm_gbs"]
    i8 = peaks["bf16_tflops"] * INT8_PER_BF16
    kern = []
    for li, stt in enumerate(stats):
        name = inputs[li].spec.name
        kern.append(dict(kernel="quantize", layer=name, ms=k1_ms[li], bound="hbm",
                         achieved=stt["k1_bytes"] / (k1_ms[li] * 1e-3) / 1e9, peak=hbm, unit="GB/s",
                         algorithmic=stt["k1_bytes"]))
        if stt["k2_issued"] / (i8 * 1e12) >= stt["k2_bytes"] / (hbm * 1e9):
            kern.append(dict(kernel="slice_gemm", layer=name, ms=k2_ms[li], bound="tensor",
                             achieved=stt["k2_dense"] / (k2_ms[li] * 1e-3) / 1e12, peak=i8, unit="TOPS",
                             algorithmic=stt["k2_dense"]))
        else:
            kern.append(dict(kernel="slice_gemm", layer=name, ms=k2_ms[li], bound="hbm",
                             achieved=stt["k2_bytes"] / (k2_ms[li] * 1e-3) / 1e9, peak=hbm, unit="GB/s",
                             algorithmic=stt["k2_bytes"]))
    for i, k in enumerate(kern):
        k["frac"] = k["achieved"] / k["peak"]
        if spread and (k["kernel"], i // 2) in spread:
            k["ms_median"], k["ms_min"], k["ms_max"] = spread[(k["kernel"], i // 2)]
    return kern


def roofline_of(kern, peak_src):
    dom = max(kern, key=lambda k: k["ms"])
    traffic = load_traffic().get(f"{dom['kernel']}.{dom['layer']}.dram_bytes")
    return {"bound": dom["bound"], "achieved": dom["achieved"], "peak": dom["peak"], "unit": dom["unit"],
            "frac": dom["frac"], "traffic": traffic, "kernel": f"{dom['kernel']} ({dom['layer']})",
            "peak_source": (f"{peak_src} hbm_gbs" if dom["bound"] == "hbm" else
                            f"{peak_src} bf16_tflops x {INT8_PER_BF16} (nominal int8:bf16)")}


def rounded(kern):
    return [{k: (round(v, 4) if isinstance(v, float) else v) for k, v in kk.items()} for kk in kern]


# ------------------------------------------------------------ oracle timing

def oracle_step(inputs, nt: int, frac: float, stage_s=None) -> float:
    """One oracle pass over the first nt token tiles of every layer and the
    first `frac` of its output channels (quantize, int64 accumulation, fp32
    epilogue); returns the dense-equivalent ops it covered and adds each
    stage's seconds to stage_s."""
    import numpy as np
    import oracle

    ops = 0.0
    for inp in inputs:
        s = inp.spec
        rows = slice(0, 16 * nt)
        ncols = s.N if frac >= 1.0 else max(16, int(s.N * frac) // 16 * 16)
        xt, xp = inp.as_f32("x_t")[rows], inp.as_f32("x_prev")[rows]
        w = np.ascontiguousarray(inp.w_q[:ncols])
        ws = np.ascontiguousarray(inp.w_scale[:ncols])
        yp = np.ascontiguousarray(inp.as_f32("y_prev")[rows, :ncols])
        t0 = time.perf_counter()
        q = oracle.quantize(xt, xp, s.lb, s.t0, s.force_bits)
        t1 = time.perf_counter()
        acc = oracle.acc_direct(q, w)
        t2 = time.perf_counter()
        oracle.epilogue_f32(acc, q.g_ref, s.lb, ws, yp, s.dtype == "bf16")
        t3 = time.perf_counter()
        if stage_s is not None:
            stage_s["quantize"] += t1 - t0
            stage_s["gemm"] += t2 - t1
            stage_s["epilogue"] += t3 - t2
        ops += 2.0 * 16 * nt * ncols * s.K
    return ops


def oracle_calibrate(inputs, per_step: float):
    """A step size of about per_step seconds that keeps every oracle thread
    busy: at least one token tile per thread, then more tiles, or a fraction
    of the output channels when even that is too long."""
    import oracle

    threads = oracle.n_threads()
    T = min(inp.spec.M // 16 for inp in inputs)
    nt = min(T, threads)
    oracle_step(inputs, nt, 1.0)  # load and warm
    t0 = time.perf_counter()
    oracle_step(inputs, nt, 1.0)
    el = time.perf_counter() - t0
    if el <= per_step:
        return max(nt, min(T, int(nt * per_step / el))), 1.0, min(threads, nt), T
    return nt, max(per_step / el, 1e-3), min(threads, nt), T


def oracle_baseline(inputs, seconds: float):
    """The CPU oracle as it stands on the host cores: (a) all threads, on the
    first token tiles of every layer, as many as take about `seconds` (the
    whole workload when it fits), timed per stage; (b) one thread on a small
    sample.  Returns the cpu_baseline entry of the JSON line."""
    import oracle

    T = min(inp.spec.M // 16 for inp in inputs)
    threads = oracle.n_threads()
    oracle_step(inputs, min(T, threads), 1.0)  # load and warm
    t0 = time.perf_counter()
    oracle_step(inputs, min(T, threads), 1.0)
    probe = time.perf_counter() - t0
    nt = max(min(T, threads), min(T, int(min(T, threads) * seconds / max(probe, 1e-6))))
    stages = {"quantize": 0.0, "gemm": 0.0, "epilogue": 0.0}
    t0 = time.perf_counter()
    ops = oracle_step(inputs, nt, 1.0, stages)
    el = time.perf_counter() - t0
    # one thread: a few token tiles of every layer
    nt1 = max(1, min(T, 4))
    stages1 = {"quantize": 0.0, "gemm": 0.0, "epilogue": 0.0}
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        ops1 = oracle_step(inputs, nt1, 1.0, stages1)
        el1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(threads)
    sample = (f"{'the whole workload' if nt == T else f'the first {nt} of {T} token tiles of every layer'} "
              f"(quantize, direct int64 accumulation, fp32 epilogue) once, {threads} threads")
    return {"value": ops / el / 1e12, "unit": "TOPS", "cores": min(threads, nt), "kind": "oracle",
            "sample": sample, "seconds": el, "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "stages_s": {k: round(v, 4) for k, v in stages.items()},
            "single_thread": {"value": ops1 / el1 / 1e12, "unit": "TOPS", "cores": 1, "seconds": el1,
                              "sample": f"the first {nt1} token tiles of every layer",
                              "stages_s": {k: round(v, 4) for k, v in stages1.items()}}}


# ----------------------------------------------------------------- arms

def run_reference(args, rank, world):
    """The oracle as the reference arm: rank 0 times it on the host cores."""
    if rank != 0:
        return
    inputs = workload_inputs(args.config, 0)
    budget = 150.0  # seconds for warmup + steps
    per_step = budget / max(1, args.steps + args.warmup)
    nt, frac, threads, T = oracle_calibrate(inputs, per_step)
    for _ in range(args.warmup):
        oracle_step(inputs, nt, frac)
    t0 = time.perf_counter()
    ops = 0.0
    for _ in range(args.steps):
        ops += oracle_step(inputs, nt, frac)
    el = time.perf_counter() - t0
    val = ops / el / 1e12
    sample = (f"{nt} of {T} token tiles x {frac:.3f} of the output channels of every layer per step "
              f"(oracle: quantize, int64 accumulation, fp32 epilogue)")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
        "config": workload_config(args.config, inputs, world, args.xprev),
        "cpu_baseline": {"value": val, "unit": "TOPS", "cores": threads, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model()},
        "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class ConfigBench:
    """One workload on this GPU: rotating input sets, CUDA graphs of the step
    (one dstar_fmdq_linear call per layer) and of the same step split into its
    two stages with event nodes between the kernels."""

    def __init__(self, cfg, args, rank, torch, nat, L):
        import numpy as np
        self.cfg, self.args, self.torch, self.nat, self.L = cfg, args, torch, nat, L
        self.inputs = workload_inputs(cfg, rank)
        self.swap = args.xprev == "swap"
        self.nsets = args.sets
        self.sets = [[Layer(inp, torch, nat, self.swap) for inp in self.inputs] for _ in range(self.nsets)]
        self.nlayers = len(self.inputs)
        self.stream = torch.cuda.current_stream()
        self.sh = ctypes.c_void_p(self.stream.cuda_stream)
        self.uses = [0] * self.nsets
        self.graphs = self.prof_graphs = self.cycle = self.gev = None
        self.np = np

    def set_mb(self):
        return sum(t.numel() * t.element_size() for lay in self.sets[0] for t in lay.tensors()) / 1e6

    def step(self, s):
        r = s % self.nsets
        parity = self.uses[r] & 1
        self.uses[r] += 1
        for lay in self.sets[r]:
            if lay.linear(self.L, parity, self.sh):
                raise RuntimeError(self.L.dstar_fmdq_last_error().decode())

    def warm_and_stats(self, warmup):
        """Untimed warm-up steps, then the workload statistics of one call per layer."""
        np = self.np
        for s in range(max(warmup, 3)):
            self.step(s)
        self.torch.cuda.synchronize()
        stats = []
        for lay in self.sets[0]:
            sec = lay.ws.sections(lay.spec.M, lay.spec.K)
            b1 = algorithmic_k1_bytes(lay.spec, sec, refresh=not self.swap)
            dense, issued, b2, nfall = algorithmic_k2(lay.spec, sec)
            bits = sec["bits"].cpu().numpy()
            planes = sec["planes"].cpu().numpy()
            # the paper's unit of MPU work: one 2-bit slice of 16 tokens against one weight
            slice_macs = 16 * int(sec["count"].cpu().numpy().astype(np.int64).sum()) * lay.spec.N
            stats.append(dict(k1_bytes=b1, k2_dense=dense, k2_issued=issued, k2_bytes=b2, fallback_tiles=nfall,
                              slice_macs=slice_macs, bits_avg=float(bits.mean()),
                              bit_hist=[float((bits == b).mean()) for b in (2, 4, 6, 8)],
                              planes_hist=[int((planes == p).sum()) for p in (1, 2)] + [int((planes > 2).sum())]))
        self.stats = stats
        return stats

    def capture(self):
        """Graphs: per (set, parity) the step and its split form, and one graph
        holding a whole cycle of steps (every set with both X_t)."""
        torch, L = self.torch, self.L
        from cuda.bindings import runtime as rt
        self.rt = rt

        def ext_event():
            err, e = rt.cudaEventCreate()
            assert err == rt.cudaError_t.cudaSuccess
            return e

        kinds = [(r, par) for par in (0, 1) for r in range(self.nsets)]
        self.gev = [[[ext_event() for _ in range(3)] for _ in range(self.nlayers)] for _ in kinds]
        self.graphs, self.prof_graphs = [], []
        cap_stream = torch.cuda.Stream()
        for gi, (r, par) in enumerate(kinds):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream):
                csh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
                for lay in self.sets[r]:
                    if lay.linear(L, par, csh):
                        raise RuntimeError(L.dstar_fmdq_last_error().decode())
            self.graphs.append(g)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream):
                cs = torch.cuda.current_stream()
                csh = ctypes.c_void_p(cs.cuda_stream)
                rsh = rt.cudaStream_t(init_value=cs.cuda_stream)
                for li, lay in enumerate(self.sets[r]):
                    rt.cudaEventRecordWithFlags(self.gev[gi][li][0], rsh, rt.cudaEventRecordExternal)
                    rc = lay.quantize(L, par, csh)
                    rt.cudaEventRecordWithFlags(self.gev[gi][li][1], rsh, rt.cudaEventRecordExternal)
                    rc |= lay.gemm(L, csh)
                    rt.cudaEventRecordWithFlags(self.gev[gi][li][2], rsh, rt.cudaEventRecordExternal)
                    if rc:
                        raise RuntimeError(L.dstar_fmdq_last_error().decode())
            self.prof_graphs.append(g)
        self.cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.cycle, stream=cap_stream):
            csh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
            for r, par in kinds:
                for lay in self.sets[r]:
                    if lay.linear(L, par, csh):
                        raise RuntimeError(L.dstar_fmdq_last_error().decode())
        for g in self.graphs:  # warm the graphs (keeps every set's parity alternating)
            g.replay()
        self.cycle.replay()
        torch.cuda.synchronize()

    def replay(self, K):
        """K steps: whole cycles, then the first steps of one."""
        n = len(self.graphs)
        for _ in range(K // n):
            self.cycle.replay()
        for s in range(K % n):
            self.graphs[s].replay()

    def split_times(self, K):
        """Per-kernel times from replays of the split step (event nodes): the
        mean over the last back-to-back cycle of every graph, returned, and in
        self.split_stats the median, min and max over 10 more cycles whose
        events are read after each replay."""
        torch, rt = self.torch, self.rt
        n = len(self.graphs)
        kp = max(n, min(K, 1200) // n * n)
        torch.cuda.synchronize()
        for s in range(kp):
            self.prof_graphs[s % n].replay()
        torch.cuda.synchronize()

        def el(a, b):
            err, v = rt.cudaEventElapsedTime(a, b)
            assert err == rt.cudaError_t.cudaSuccess
            return v
        k1 = [statistics.fmean(el(self.gev[g][li][0], self.gev[g][li][1]) for g in range(n))
              for li in range(self.nlayers)]
        k2 = [statistics.fmean(el(self.gev[g][li][1], self.gev[g][li][2]) for g in range(n))
              for li in range(self.nlayers)]
        samples = {}
        for _ in range(10):
            for g in range(n):
                self.prof_graphs[g].replay()
                torch.cuda.synchronize()
                for li in range(self.nlayers):
                    samples.setdefault(("quantize", li), []).append(el(self.gev[g][li][0], self.gev[g][li][1]))
                    samples.setdefault(("slice_gemm", li), []).append(el(self.gev[g][li][1], self.gev[g][li][2]))
        self.split_stats = {k: (statistics.median(v), min(v), max(v)) for k, v in samples.items()}
        return k1, k2

    def timed(self, K, dist=False, clocks_id=None, clocks_on=True):
        """Device time of K steps (CUDA events, barrier + synchronize around)."""
        torch = self.torch
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks = ClockSampler(clocks_id, clocks_on) if clocks_id is not None else None
        if clocks is not None:
            time.sleep(0.3)
        if dist:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t_wall0 = time.time()
        ev0.record(self.stream)
        if self.graphs:
            self.replay(K)
        else:
            for s in range(K):
                self.step(s)
        ev1.record(self.stream)
        torch.cuda.synchronize()
        t_wall1 = time.time()
        if dist:
            torch.distributed.barrier()
        clock_summary = None
        if clocks is not None:
            time.sleep(0.2)
            clocks.stop()
            clock_summary = clocks.summary(t_wall0, t_wall1)
        return ev0.elapsed_time(ev1), clock_summary

    def e2e(self, steps, world, dense_step):
        """The same metric through the public API with host buffers: per step
        X_t of every layer copied in from pinned host memory, the calls, Y_t
        of every layer copied back.  Copies run on their own streams; a set's
        landing buffers are rewritten only after that set's previous compute
        finished, and its Y cache updated only after that set's previous
        read-back finished."""
        torch, L, nat = self.torch, self.L, self.nat
        sets, swap, stream, sh = self.sets, self.swap, self.stream, self.sh
        host_x = [[[torch.empty_like(lay.x_a, device="cpu").pin_memory() for _ in range(2)] for lay in st]
                  for st in sets]
        host_y = [[torch.empty_like(lay.y_prev, device="cpu").pin_memory() for lay in st] for st in sets]
        for r, st in enumerate(sets):
            for li, lay in enumerate(st):
                host_x[r][li][0].copy_(lay.x_a.cpu())
                host_x[r][li][1].copy_(lay.x_b.cpu())
        h2d = sum(lay.x_a.numel() * lay.x_a.element_size() for lay in sets[0])
        d2h = sum(lay.y_prev.numel() * lay.y_prev.element_size() for lay in sets[0])
        # device landing buffers: one per parity in swap mode (the other
        # parity's buffer holds X_{t-1}), else one
        land = [[[lay.x_a.clone(), lay.x_b.clone()] if swap else [torch.empty_like(lay.x_a)] for lay in st]
                for st in sets]
        land_m = [[[nat.mat(t) for t in bufs] for bufs in row] for row in land]
        h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
        last_c = [None] * self.nsets  # per set: its last compute, its last read-back
        last_d = [None] * self.nsets

        def step_e2e(s):
            r = s % self.nsets
            parity = self.uses[r] & 1
            self.uses[r] += 1
            slot = parity if swap else 0
            if last_c[r] is not None:
                h2d_s.wait_event(last_c[r])
            with torch.cuda.stream(h2d_s):
                for li in range(len(sets[r])):
                    land[r][li][slot].copy_(host_x[r][li][parity], non_blocking=True)
            ev_h = torch.cuda.Event()
            ev_h.record(h2d_s)
            stream.wait_event(ev_h)
            if last_d[r] is not None:
                stream.wait_event(last_d[r])
            for li, lay in enumerate(sets[r]):
                mp = land_m[r][li][1 - parity] if swap else lay.m_xp
                rc = L.dstar_fmdq_linear(ctypes.byref(land_m[r][li][slot]), ctypes.byref(mp), ctypes.byref(lay.m_y),
                                         ctypes.byref(lay.m_w), lay.ws_ptr, lay.base, ctypes.byref(lay.cfg),
                                         ctypes.byref(lay.m_y), sh)
                if rc:
                    raise RuntimeError(L.dstar_fmdq_last_error().decode())
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            last_c[r] = ev_c
            d2h_s.wait_event(ev_c)
            with torch.cuda.stream(d2h_s):
                for li, lay in enumerate(sets[r]):
                    host_y[r][li].copy_(lay.y_prev, non_blocking=True)
            ev_d = torch.cuda.Event()
            ev_d.record(d2h_s)
            last_d[r] = ev_d

        for s in range(3):
            step_e2e(s)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(h2d_s)
        for s in range(steps):
            step_e2e(s)
        stream.wait_stream(h2d_s)
        stream.wait_stream(d2h_s)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), "cuda")
        return {"value": job_tops(world, dense_step, ems / steps), "unit": "TOPS", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ems / steps,
                "path": "pinned host X_t -> device, dstar_fmdq_linear per layer, Y_t -> pinned host; copies on "
                        "their own streams overlap the neighbouring steps' compute"}

    def status(self):
        st = 0
        for row in self.sets:
            for lay in row:
                st |= self.nat.status(lay.ws)
        return st

    def close(self):
        self.graphs = self.prof_graphs = self.cycle = None
        self.sets = None
        self.torch.cuda.synchronize()
        self.torch.cuda.empty_cache()


def measure_extra(cfg, args, torch, nat, L, peaks, peak_src):
    """A further workload on this GPU: step time, per-kernel times, roofline
    and workload statistics (no e2e, no clocks)."""
    from differential_quantized_gemm_b200 import synth
    cb = ConfigBench(cfg, args, 0, torch, nat, L)
    stats = cb.warm_and_stats(args.warmup)
    cb.capture()
    ms, _ = cb.timed(args.extra_steps)
    k1, k2 = cb.split_times(args.extra_steps)
    st = cb.status()
    if st:
        raise RuntimeError(f"device status {st} after workload {cfg}")
    dense = sum(s["k2_dense"] for s in stats)
    kern = kernel_rows(cb.inputs, stats, k1, k2, peaks, getattr(cb, "split_stats", None))
    out = {"workload": synth.CONFIG_NAMES[cfg], "value": job_tops(1, dense, ms / args.extra_steps), "unit": "TOPS",
           "ms_per_step": ms / args.extra_steps, "steps": args.extra_steps,
           "layers": [f"{i.spec.name} M={i.spec.M} K={i.spec.K} N={i.spec.N}" for i in cb.inputs],
           "roofline": roofline_of(kern, peak_src), "kernels": rounded(kern),
           "workload_stats": [{k: v for k, v in s.items() if k in ("bits_avg", "bit_hist", "planes_hist",
                                                                 "fallback_tiles", "slice_macs")} for s in stats]}
    cb.close()
    return out


def measure_sweep(args, torch, nat, L):
    """The 28-layer DiT-XL stack over the timestep sweep: 50 steps with every
    layer's caches carried from step to step (X_t = X_{t-1} + sigma_t N(0, 1),
    sigma_t U-shaped), then the forced all-2-bit and all-8-bit runs at
    sigma 0.03.  Before each step (untimed) the new X_t of all 56 calls is
    drawn on the device from a seeded generator; the step itself (56
    dstar_fmdq_linear calls replayed from one CUDA graph) is timed with events."""
    from differential_quantized_gemm_b200 import synth
    specs = synth.config_layers(5)
    nl = len(specs)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    xs, xn, ys, wq, wsc, wss, cfgs = [], [], [], [], [], [], {0: [], 2: [], 8: []}
    for li, sp in enumerate(specs):
        w, sc = synth.layer_weights(5, li)
        wq.append(torch.from_numpy(w).cuda())
        wsc.append(torch.from_numpy(sc).cuda())
        x0 = torch.randn(sp.M, sp.K, generator=gen, device="cuda").to(torch.bfloat16)
        xs.append(x0)                         # x_prev cache, refreshed by the quantizer
        xn.append(torch.empty_like(x0))      # X_t of the step
        # step-0 dense initialisation of the cached output (not timed): Y = X W_deq
        wdeq = wq[-1].float().t() * wsc[-1][None, :]
        ys.append((x0.float() @ wdeq).to(torch.bfloat16))
        ws = nat.Workspace(sp.M, sp.K)
        wss.append(ws)
        for fb in cfgs:
            cfgs[fb].append(nat.TileCfg(16, sp.t0, fb, 0, ctypes.c_void_p(ws.ptr), ws.nbytes, None, None))
    m_xn = [nat.mat(t) for t in xn]
    m_xs = [nat.mat(t) for t in xs]
    m_y = [nat.mat(t) for t in ys]
    m_w = [nat.mat(t) for t in wq]
    base = 2.0 ** specs[0].lb
    zbuf = torch.empty(max(sp.M * sp.K for sp in specs), device="cuda")

    def draw(sigma):
        for li, sp in enumerate(specs):
            z = zbuf[:sp.M * sp.K].view(sp.M, sp.K)
            torch.randn(sp.M, sp.K, generator=gen, out=z)
            xn[li].copy_((xs[li].float() + sigma * z).to(torch.bfloat16))

    graphs = {}
    cap = torch.cuda.Stream()
    for fb in cfgs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            csh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
            for li in range(nl):
                rc = L.dstar_fmdq_linear(ctypes.byref(m_xn[li]), ctypes.byref(m_xs[li]), ctypes.byref(m_y[li]),
                                         ctypes.byref(m_w[li]), ctypes.c_void_p(wsc[li].data_ptr()), base,
                                         ctypes.byref(cfgs[fb][li]), ctypes.byref(m_y[li]), csh)
                if rc:
                    raise RuntimeError(L.dstar_fmdq_last_error().decode())
        graphs[fb] = g
    dense_step = sum(2.0 * sp.M * sp.N * sp.K for sp in specs)
    stream = torch.cuda.current_stream()

    def layer_stats():
        bits_sum = torch.zeros((), dtype=torch.float64, device="cuda")
        n = 0
        ph = torch.zeros(3, dtype=torch.int64, device="cuda")
        for li, sp in enumerate(specs):
            sec = wss[li].sections(sp.M, sp.K)
            bits_sum += sec["bits"].double().sum()
            n += sec["bits"].numel()
            pl = sec["planes"].long()
            ph += torch.stack([(pl == 1).sum(), (pl == 2).sum(), (pl > 2).sum()])
        return bits_sum, n, ph

    def run(fb, sigma_of, nsteps):
        ms, bits, planes = [], [], []
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nsteps)]
        pend = []
        for t in range(nsteps):
            draw(sigma_of(t))
            ev[t][0].record(stream)
            graphs[fb].replay()
            ev[t][1].record(stream)
            pend.append(layer_stats())
        torch.cuda.synchronize()
        for t in range(nsteps):
            ms.append(ev[t][0].elapsed_time(ev[t][1]))
            bsum, n, ph = pend[t]
            bits.append(float(bsum.item()) / n)
            planes.append([int(v) for v in ph.cpu()])
        return ms, bits, planes

    draw(synth.sweep_sigma(0))  # warm the graphs on a throw-away step of each kind (caches advance)
    for fb in cfgs:
        graphs[fb].replay()
    torch.cuda.synchronize()
    steps = args.sweep_steps
    ms, bits, planes = run(0, synth.sweep_sigma, steps)
    out = {"workload": synth.CONFIG_NAMES[5], "layers": nl, "M": specs[0].M, "steps": steps,
           "timing": "each step: 56 dstar_fmdq_linear calls replayed from one CUDA graph, CUDA events around "
                     "it; the step's X_t are drawn on the device before it (untimed)",
           "ms_per_step": [round(v, 4) for v in ms], "ms_per_step_mean": statistics.fmean(ms),
           "value": dense_step / (statistics.fmean(ms) * 1e-3) / 1e12, "unit": "TOPS",
           "bits_avg_per_step": [round(b, 3) for b in bits],
           "planes_hist_per_step": planes, "fallback_tiles_total": int(sum(p[2] for p in planes))}
    for fb, key in ((2, "forced_2bit"), (8, "forced_8bit")):
        ms_f, bits_f, planes_f = run(fb, lambda t: 0.03, args.extreme_reps)
        out[key] = {"ms_per_step_mean": statistics.fmean(ms_f),
                    "value": dense_step / (statistics.fmean(ms_f) * 1e-3) / 1e12, "unit": "TOPS",
                    "bits_avg": bits_f[-1], "planes_hist": planes_f[-1], "fallback_tiles": planes_f[-1][2],
                    "vs_adaptive_mean_step": statistics.fmean(ms_f) / statistics.fmean(ms), "reps": args.extreme_reps}
    st = 0
    for ws in wss:
        st |= nat.status(ws)
    if st:
        raise RuntimeError(f"device status {st} after the sweep")
    del graphs
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def measure_dyn(args, torch, nat, L):
    """The headline workload with the dynamic base (FMDQ-DYN): a first pass
    finds min M_i, then the same quantizer and GEMM."""
    cb = ConfigBench(args.config, args, 0, torch, nat, L)
    for row in cb.sets:
        for lay in row:
            lay.cfg.flags |= nat.FLAG_DYNAMIC_BASE
    stats = cb.warm_and_stats(args.warmup)
    cb.capture()
    steps = args.extra_steps
    ms, _ = cb.timed(steps)
    k1, k2 = cb.split_times(steps)
    st = cb.status()
    if st:
        raise RuntimeError(f"device status {st} after the dynamic-base run")
    dense = sum(s_["k2_dense"] for s_ in stats)
    bases = [float(lay.ws.sections(lay.spec.M, lay.spec.K)["dyn_base"].cpu()[0]) for lay in cb.sets[0]]
    out = {"what": "FMDQ-DYN (dynamic base = min M_i of the call, found by a first pass over X_t, X_{t-1})",
           "value": job_tops(1, dense, ms / steps), "unit": "TOPS", "ms_per_step": ms / steps, "steps": steps,
           "kernels": [{"layer": i.spec.name, "quantize_ms": round(a, 4), "slice_gemm_ms": round(b, 4)}
                       for i, a, b in zip(cb.inputs, k1, k2)],
           "bits_avg": [s_["bits_avg"] for s_ in stats], "dynamic_base": bases,
           "gpu_launches_per_step": 3 * len(cb.inputs)}
    cb.close()
    return out


def measure_ffn_gelu(args, torch, nat, L):
    """The chained FFN pair of the headline workload with the GELU fused into
    the first layer's epilogue (dstar_fmdq_ffn_gelu): X_t alternates between two
    draws; every cache (x_prev, Y1, H, Y2) is carried by the library."""
    from differential_quantized_gemm_b200 import synth
    up = synth.make_layer(args.config, 0)
    w2, s2 = synth.layer_weights(args.config, 1)
    dev = "cuda"

    def bf(a):
        return torch.from_numpy(a).view(torch.bfloat16).to(dev)

    xa, xb = bf(up.x_t), bf(up.x_prev)
    x_prev = xb.clone()
    y1 = bf(up.y_prev)
    # H_{t-1} = GELU(Y1_{t-1}) and Y2_{t-1} = H_{t-1} W2_deq: the dense state of step 0 (not timed)
    h_prev = torch.nn.functional.gelu(y1.float()).to(torch.bfloat16)
    w1, ws1 = torch.from_numpy(up.w_q).to(dev), torch.from_numpy(up.w_scale).to(dev)
    w2t, ws2 = torch.from_numpy(w2).to(dev), torch.from_numpy(s2).to(dev)
    y2 = (h_prev.float() @ (w2t.float().t() * ws2[None, :])).to(torch.bfloat16)
    h_t = torch.empty_like(h_prev)
    M, K1, N1 = up.spec.M, up.spec.K, up.spec.N
    wsa, wsb = nat.Workspace(M, K1), nat.Workspace(M, N1)
    base = 2.0 ** up.spec.lb
    stream = torch.cuda.current_stream()
    graphs = []
    cap = torch.cuda.Stream()
    for x in (xa, xb):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            nat.ffn_gelu(x, x_prev, y1, w1, ws1, h_t, h_prev, y2, w2t, ws2, base, wsa, wsb)
        graphs.append(g)
    for _ in range(max(args.warmup, 4)):
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    steps = args.extra_steps // 2 * 2
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        graphs[i % 2].replay()
    e1.record(stream)
    torch.cuda.synchronize()
    if nat.status(wsa) or nat.status(wsb):
        raise RuntimeError("device status after the chained FFN pair")
    ms = e0.elapsed_time(e1) / steps
    layer_stats = []
    for ws, K in ((wsa, K1), (wsb, N1)):
        sec = ws.sections(M, K)
        bits, planes = sec["bits"].float(), sec["planes"]
        layer_stats.append({"bits_avg": float(bits.mean()),
                            "planes_hist": [int((planes == 1).sum()), int((planes == 2).sum()),
                                            int((planes > 2).sum())]})
    dense = 2.0 * M * N1 * K1 + 2.0 * M * w2.shape[0] * N1
    del graphs
    torch.cuda.synchronize()
    return {"what": "chained FFN pair, GELU fused into the first layer's epilogue (dstar_fmdq_ffn_gelu)",
            "workload": synth.CONFIG_NAMES[args.config], "value": dense / (ms * 1e-3) / 1e12, "unit": "TOPS",
            "ms_per_step": ms, "steps": steps, "gpu_launches_per_step": 4,
            "layer_stats": layer_stats,
            "note": "layer 2 quantizes the differential of GELU(Y1), wider than the independent draw of the "
                    "headline's second layer (more 8-bit sub-channels and two-plane tiles)"}


def measure_sar(args, torch, nat, L):
    """Sparse attention reuse with INT8 FMDQ operands on the PixArt 1024px
    attention: 2 x 16 heads of 4096 tokens, head dimension 72 (padded to 96),
    a synthetic block mask keeping every diagonal block and half of the
    others, the scores recomputed every second step (interval 2)."""
    import math
    from differential_quantized_gemm_b200 import synth
    G, S, dh, d = 32, 4096, 72, 96
    qb, kb, vb, v2b, mask = synth.attention_inputs(G, S, dh, d, seed=11, keep=0.5)

    def dev(b):
        return torch.from_numpy(b).view(torch.bfloat16).cuda()

    q, k, v, v2 = dev(qb), dev(kb), dev(vb), dev(v2b)
    out = torch.empty(G * S, d, dtype=torch.float32, device="cuda")
    att = nat.SarAttention(G, S, d, mask, float(1.0 / math.sqrt(dh)), 2.0 ** -4, 2.0 ** -6)
    stream = torch.cuda.current_stream()
    cap = torch.cuda.Stream()
    g_cached, g_reused = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_cached, stream=cap):
        att(q, k, v, out)
    with torch.cuda.graph(g_reused, stream=cap):
        att(q, k, v2, out, reuse=True)
    for _ in range(3):
        g_cached.replay()
        g_reused.replay()
    torch.cuda.synchronize()
    reps = max(4, min(40, args.extra_steps // 30))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    tc, tr = [], []
    for _ in range(reps):
        ev[0].record(stream)
        g_cached.replay()
        ev[1].record(stream)
        g_reused.replay()
        ev[2].record(stream)
        torch.cuda.synchronize()
        tc.append(ev[0].elapsed_time(ev[1]))
        tr.append(ev[1].elapsed_time(ev[2]))
    if att.status():
        raise RuntimeError("device status after the attention run")
    kept = float(mask.mean())
    dense = 4.0 * G * S * S * dh  # Q K^T and P V of full attention at the unpadded head dimension
    c, r = statistics.median(tc), statistics.median(tr)
    del g_cached, g_reused
    torch.cuda.synchronize()
    return {"what": "sparse attention reuse, INT8 FMDQ operands (dstar_sar_attention)",
            "workload": f"PixArt 1024px attention: {G} heads x {S} tokens, head dim {dh} (padded to {d}), "
                        f"{kept:.3f} of the 128x128 blocks kept, interval 2",
            "cached_step_ms": c, "reused_step_ms": r, "ms_per_step": (c + r) / 2,
            "value": dense / ((c + r) / 2 * 1e-3) / 1e12, "unit": "dense-equivalent attention TOPS",
            "kept_block_fraction": kept, "reps": reps, "gpu_launches_per_step": 4.5}


def run_ours(args, rank, world, local_rank):
    import torch

    from differential_quantized_gemm_b200 import _native as nat
    from differential_quantized_gemm_b200 import build as cuda_build

    if rank == 0:
        cuda_build.build()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.set_device(local_rank)
    L = nat.lib()
    dist = world > 1
    peaks, peak_src = load_peaks()

    cb = ConfigBench(args.config, args, rank, torch, nat, L)
    stats = cb.warm_and_stats(args.warmup)
    K = args.steps
    if args.mode == "graph":
        cb.capture()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_id = vis.split(",")[local_rank] if vis else str(torch.cuda.current_device())
    ms, clocks = cb.timed(K, dist, smi_id, not args.no_clocks)
    if cb.graphs:
        k1_ms, k2_ms = cb.split_times(K)
    else:  # eager: one more pass with events around each stage
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(cb.nlayers)]
        k1_ms, k2_ms = [0.0] * cb.nlayers, [0.0] * cb.nlayers
        for s in range(K):
            r = s % cb.nsets
            parity = cb.uses[r] & 1
            cb.uses[r] += 1
            for li, lay in enumerate(cb.sets[r]):
                evs[li][0].record(cb.stream)
                lay.quantize(L, parity, cb.sh)
                evs[li][1].record(cb.stream)
                lay.gemm(L, cb.sh)
                evs[li][2].record(cb.stream)
            torch.cuda.synchronize()
            for li in range(cb.nlayers):
                k1_ms[li] += evs[li][0].elapsed_time(evs[li][1]) / K
                k2_ms[li] += evs[li][1].elapsed_time(evs[li][2]) / K
    ms = max_over_ranks(ms, "cuda")
    ms_step = ms / K
    dense_step = sum(st["k2_dense"] for st in stats)
    value = job_tops(world, dense_step, ms_step)
    e2e = cb.e2e(min(args.e2e_steps, K), world, dense_step)
    st = cb.status()
    if st:
        raise RuntimeError(f"device status {st} after the benchmark")
    inputs = cb.inputs
    set_mb = cb.set_mb()
    spread = getattr(cb, "split_stats", None)
    cb.close()

    # further workloads, on one GPU only (every rank would have to run them alike)
    per_config, sweep, next_rows = [], None, None
    if world == 1:
        for c in [int(x) for x in args.extra_configs.split(",") if x.strip()]:
            if c != args.config:
                per_config.append(measure_extra(c, args, torch, nat, L, peaks, peak_src))
        if args.sweep_steps > 0:
            sweep = measure_sweep(args, torch, nat, L)
        if not args.no_next_rows:
            next_rows = {"ffn_gelu": measure_ffn_gelu(args, torch, nat, L),
                         "dynamic_base": measure_dyn(args, torch, nat, L),
                         "sar_attention": measure_sar(args, torch, nat, L)}

    if rank != 0:
        return

    kern = kernel_rows(inputs, stats, k1_ms, k2_ms, peaks, spread)
    roofline = roofline_of(kern, peak_src)
    cpu = None
    if not args.no_cpu_baseline:
        cpu = oracle_baseline(inputs, args.cpu_seconds)

    nlayers = len(inputs)
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": dict(workload_config(args.config, inputs, world, args.xprev),
                       l2=f"inputs rotate over {args.sets} buffer sets of {set_mb:.0f} MB each "
                          f"({args.sets * set_mb:.0f} MB > 126 MB L2); no flush needed"),
        "roofline": roofline,
        "kernels": rounded(kern),
        "quantizer_GBps": [k["achieved"] for k in kern if k["kernel"] == "quantize"],
        "quantizer_frac_of_8TBs_spec": [k["achieved"] / 8000.0 for k in kern if k["kernel"] == "quantize"],
        "workload_stats": [{k: v for k, v in s.items() if k in ("bits_avg", "bit_hist", "planes_hist",
                                                              "fallback_tiles", "slice_macs")} for s in stats],
        "slice_macs_per_s": sum(s["slice_macs"] for s in stats) / (ms_step * 1e-3),
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": 2 * nlayers * K,
        "clocks": clocks,
        "per_config": per_config, "sweep": sweep, "next_rows": next_rows,
        "kernel_sources": kernel_source_sha(),
        "timing": ("value: CUDA-graph replays of the captured dstar_fmdq_linear calls, one graph per cycle of "
                   f"{2 * args.sets} steps (every input set with both X_t); per-kernel times: a second timed "
                   "region of the step split into dstar_fmdq_quantize + dstar_fmdq_slice_gemm with event nodes "
                   "between the kernels" if args.mode == "graph"
                   else "eager C-ABI calls; per-kernel times from events around each stage"),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
