#!/usr/bin/env python
"""Benchmark of the FMDQ differential linear hot path on B200.

One step = one pass of the whole hot path over one batch: for every layer of
the workload, the quantizer (K1) and the slice GEMM with its fused epilogue
(K2, plus the slice-stream kernel for tiles that need it), through the C ABI.
Default workload: the DiT-XL/2 256px FFN pair, batch 8 x 256 tokens,
1152 -> 4608 -> 1152, bf16 activations, int8 weights.

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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=2, help="workload (2: DiT-XL/2 FFN pair)")
    ap.add_argument("--sets", type=int, default=3, help="rotating input sets (together larger than L2)")
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--xprev", choices=["swap", "copy"], default="copy",
                    help="swap: X_t and X_{t-1} stay resident and trade buffers each step (no refresh copy); "
                         "copy: the quantizer copies X_t into one x_prev cache")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--mode", choices=["graph", "eager"], default="graph",
                    help="graph: each step replays a captured CUDA graph; eager: C-ABI calls per step")
    return ap.parse_args()


# ----------------------------------------------------------------- peaks

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "differential_quantized_gemm_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
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


# ------------------------------------------------------------ oracle timing

def oracle_step(inputs, nt: int, frac: float) -> float:
    """One oracle pass over the first nt token tiles of every layer and the
    first `frac` of its output channels (quantize, int64 accumulation, fp32
    epilogue); returns the dense-equivalent ops it covered."""
    import numpy as np
    import oracle

    ops = 0.0
    for inp in inputs:
        s = inp.spec
        rows = slice(0, 16 * nt)
        ncols = s.N if frac >= 1.0 else max(16, int(s.N * frac) // 16 * 16)
        q = oracle.quantize(inp.as_f32("x_t")[rows], inp.as_f32("x_prev")[rows], s.lb, s.t0, s.force_bits)
        acc = oracle.acc_direct(q, np.ascontiguousarray(inp.w_q[:ncols]))
        oracle.epilogue_f32(acc, q.g_ref, s.lb, np.ascontiguousarray(inp.w_scale[:ncols]),
                            np.ascontiguousarray(inp.as_f32("y_prev")[rows, :ncols]), s.dtype == "bf16")
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


def oracle_sample_time(inputs, seconds: float):
    """Time the CPU oracle on the whole workload (every token tile of every
    layer), repeated until about `seconds`; returns (ops, elapsed,
    description, threads used)."""
    import oracle

    T = min(inp.spec.M // 16 for inp in inputs)
    oracle_step(inputs, min(T, oracle.n_threads()), 1.0)  # load and warm
    ops = el = 0.0
    reps = 0
    while reps == 0 or (el < seconds and reps < 100):
        t0 = time.perf_counter()
        ops += oracle_step(inputs, T, 1.0)
        el += time.perf_counter() - t0
        reps += 1
    desc = (f"the whole workload ({T} token tiles of every layer) {reps} time(s): quantize, direct int64 "
            f"accumulation, fp32 epilogue")
    return ops, el, desc, min(oracle.n_threads(), T)


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
    from differential_quantized_gemm_b200 import synth
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
        "config": workload_config(args.config, inputs, world, args.xprev),
        "cpu_baseline": {"value": val, "unit": "TOPS", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    from differential_quantized_gemm_b200 import _native as nat
    from differential_quantized_gemm_b200 import build as cuda_build
    from differential_quantized_gemm_b200 import synth

    if rank == 0:
        cuda_build.build()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.set_device(local_rank)
    L = nat.lib()
    dist = world > 1

    inputs = workload_inputs(args.config, rank)
    swap = args.xprev == "swap"
    sets = [[Layer(inp, torch, nat, swap) for inp in inputs] for _ in range(args.sets)]
    nlayers = len(inputs)
    stream = torch.cuda.current_stream()
    sh = ctypes.c_void_p(stream.cuda_stream)
    uses = [0] * args.sets

    def step(s, evs=None):
        r = s % args.sets
        parity = uses[r] & 1
        uses[r] += 1
        for li, lay in enumerate(sets[r]):
            if evs is not None:
                evs[li][0].record(stream)
            rc = lay.quantize(L, parity, sh)
            if evs is not None:
                evs[li][1].record(stream)
            rc |= lay.gemm(L, sh)
            if evs is not None:
                evs[li][2].record(stream)
            if rc:
                raise RuntimeError(L.dstar_fmdq_last_error().decode())

    # warm-up (untimed) and the workload statistics of one call per layer
    for s in range(max(args.warmup, 3)):
        step(s)
    torch.cuda.synchronize()
    stats = []
    for lay in sets[0]:
        sec = lay.ws.sections(lay.spec.M, lay.spec.K)
        b1 = algorithmic_k1_bytes(lay.spec, sec, refresh=not swap)
        dense, issued, b2, nfall = algorithmic_k2(lay.spec, sec)
        bits = sec["bits"].cpu().numpy()
        planes = sec["planes"].cpu().numpy()
        # the paper's unit of MPU work: one 2-bit slice of 16 tokens against one weight
        slice_macs = 16 * int(sec["count"].cpu().numpy().astype(np.int64).sum()) * lay.spec.N
        stats.append(dict(k1_bytes=b1, k2_dense=dense, k2_issued=issued, k2_bytes=b2, fallback_tiles=nfall,
                          slice_macs=slice_macs,
                          bits_avg=float(bits.mean()), bit_hist=[float((bits == b).mean()) for b in (2, 4, 6, 8)],
                          planes_hist=[int((planes == p).sum()) for p in (1, 2)] + [int((planes > 2).sum())]))

    # timed region
    K = args.steps
    graphs, gev = None, None
    if args.mode == "graph":
        # one graph per (input set, parity); each holds the step's launches and
        # external event-record nodes between them (per-kernel times)
        from cuda.bindings import runtime as rt

        def ext_event():
            err, e = rt.cudaEventCreate()
            assert err == rt.cudaError_t.cudaSuccess
            return e

        kinds = [(r, par) for par in (0, 1) for r in range(args.sets)]
        gev = [[[ext_event() for _ in range(3)] for _ in range(nlayers)] for _ in kinds]
        graphs, prof_graphs = [], []
        cap_stream = torch.cuda.Stream()
        for gi, (r, par) in enumerate(kinds):
            # the step as a user runs it: one dstar_fmdq_linear call per layer
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream):
                csh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
                for lay in sets[r]:
                    if lay.linear(L, par, csh):
                        raise RuntimeError(L.dstar_fmdq_last_error().decode())
            graphs.append(g)
            # the same step split into its two stages with event nodes between the kernels
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap_stream):
                cs = torch.cuda.current_stream()
                csh = ctypes.c_void_p(cs.cuda_stream)
                rsh = rt.cudaStream_t(init_value=cs.cuda_stream)
                for li, lay in enumerate(sets[r]):
                    rt.cudaEventRecordWithFlags(gev[gi][li][0], rsh, rt.cudaEventRecordExternal)
                    rc = lay.quantize(L, par, csh)
                    rt.cudaEventRecordWithFlags(gev[gi][li][1], rsh, rt.cudaEventRecordExternal)
                    rc |= lay.gemm(L, csh)
                    rt.cudaEventRecordWithFlags(gev[gi][li][2], rsh, rt.cudaEventRecordExternal)
                    if rc:
                        raise RuntimeError(L.dstar_fmdq_last_error().decode())
            prof_graphs.append(g)
        # the whole cycle of steps in one graph: a replay launches it once, so
        # consecutive steps follow each other without a graph launch between them
        cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cycle, stream=cap_stream):
            csh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
            for r, par in kinds:
                for lay in sets[r]:
                    if lay.linear(L, par, csh):
                        raise RuntimeError(L.dstar_fmdq_last_error().decode())
        for g in graphs:  # warm the graphs (keeps every set's parity alternating)
            g.replay()
        cycle.replay()
        torch.cuda.synchronize()
    evs = None if graphs else \
        [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nlayers)] for _ in range(K)]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_id = vis.split(",")[local_rank] if vis else str(torch.cuda.current_device())
    clocks = ClockSampler(smi_id, not args.no_clocks)
    time.sleep(0.3)
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ev0.record(stream)
    if graphs:  # step s runs graph s % len(graphs): whole cycles, then the first steps of one
        for _ in range(K // len(graphs)):
            cycle.replay()
        for s in range(K % len(graphs)):
            graphs[s].replay()
    else:
        for s in range(K):
            step(s, evs[s])
    ev1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if graphs:  # continue every set's X_t alternation after the replays (both regions)
        for s in range(K + max(len(graphs), min(K, 1200) // len(graphs) * len(graphs))):
            gi = s % len(graphs)
            uses[gi % args.sets] = gi // args.sets + 1
    if dist:
        torch.distributed.barrier()
    time.sleep(0.2)
    clocks.stop()
    ms = ev0.elapsed_time(ev1)
    if graphs:
        # per-kernel times: a second timed region of the split step, continuing
        # every set's X_t alternation; the event nodes hold each graph's last replay
        kp = max(len(graphs), min(K, 1200) // len(graphs) * len(graphs))
        torch.cuda.synchronize()
        for s in range(K, K + kp):
            prof_graphs[s % len(graphs)].replay()
        torch.cuda.synchronize()

        def el(a, b):
            err, v = rt.cudaEventElapsedTime(a, b)
            assert err == rt.cudaError_t.cudaSuccess
            return v
        k1_ms = [statistics.fmean(el(gev[g][li][0], gev[g][li][1]) for g in range(len(graphs))) for li in range(nlayers)]
        k2_ms = [statistics.fmean(el(gev[g][li][1], gev[g][li][2]) for g in range(len(graphs))) for li in range(nlayers)]
    else:
        k1_ms = [statistics.fmean(evs[s][li][0].elapsed_time(evs[s][li][1]) for s in range(K)) for li in range(nlayers)]
        k2_ms = [statistics.fmean(evs[s][li][1].elapsed_time(evs[s][li][2]) for s in range(K)) for li in range(nlayers)]
    ms = max_over_ranks(ms, "cuda")
    ms_step = ms / K
    dense_step = sum(st["k2_dense"] for st in stats)
    value = job_tops(world, dense_step, ms_step)

    # e2e: host buffers, copies inside the timed region
    e2e = None
    ke = min(args.e2e_steps, K)
    host_x = [[[torch.empty_like(lay.x_a, device="cpu").pin_memory() for _ in range(2)] for lay in st]
              for st in sets]
    host_y = [[torch.empty_like(lay.y_prev, device="cpu").pin_memory() for lay in st] for st in sets]
    for r, st in enumerate(sets):
        for li, lay in enumerate(st):
            host_x[r][li][0].copy_(lay.x_a.cpu())
            host_x[r][li][1].copy_(lay.x_b.cpu())
    h2d = sum(lay.x_a.numel() * lay.x_a.element_size() for lay in sets[0])
    d2h = sum(lay.y_prev.numel() * lay.y_prev.element_size() for lay in sets[0])
    # device landing buffers for the copied inputs: one per parity in swap
    # mode (the buffer of the other parity holds X_{t-1}), else one
    land = [[[lay.x_a.clone(), lay.x_b.clone()] if swap else [torch.empty_like(lay.x_a)] for lay in st]
            for st in sets]
    land_m = [[[nat.mat(t) for t in bufs] for bufs in row] for row in land]

    # Three streams: host->device copies, the compute (the library's calls) and
    # device->host copies, so one step's copies overlap its neighbours' compute.
    # A step's landing buffers are rewritten only after the set's previous step
    # has computed, and its Y cache is updated only after the set's previous
    # read-back has finished.
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    n_ev = ke + 3
    ev_h, ev_c, ev_d = ([torch.cuda.Event() for _ in range(n_ev)] for _ in range(3))

    def step_e2e(s, i):
        r = s % args.sets
        parity = uses[r] & 1
        uses[r] += 1
        slot = parity if swap else 0
        if i >= args.sets:
            h2d_s.wait_event(ev_c[i - args.sets])
        with torch.cuda.stream(h2d_s):
            for li in range(len(sets[r])):
                land[r][li][slot].copy_(host_x[r][li][parity], non_blocking=True)
        ev_h[i].record(h2d_s)
        stream.wait_event(ev_h[i])
        if i >= args.sets:
            stream.wait_event(ev_d[i - args.sets])
        for li, lay in enumerate(sets[r]):
            mp = land_m[r][li][1 - parity] if swap else lay.m_xp
            rc = L.dstar_fmdq_linear(ctypes.byref(land_m[r][li][slot]), ctypes.byref(mp), ctypes.byref(lay.m_y),
                                     ctypes.byref(lay.m_w), lay.ws_ptr, lay.base, ctypes.byref(lay.cfg),
                                     ctypes.byref(lay.m_y), sh)
            if rc:
                raise RuntimeError(L.dstar_fmdq_last_error().decode())
        ev_c[i].record(stream)
        d2h_s.wait_event(ev_c[i])
        with torch.cuda.stream(d2h_s):
            for li, lay in enumerate(sets[r]):
                host_y[r][li].copy_(lay.y_prev, non_blocking=True)
        ev_d[i].record(d2h_s)

    for s in range(3):
        step_e2e(s, s)
    if dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d_s)
    for s in range(ke):
        step_e2e(s, 3 + s)
    stream.wait_stream(h2d_s)
    stream.wait_stream(d2h_s)
    e1.record(stream)
    torch.cuda.synchronize()
    ems = max_over_ranks(e0.elapsed_time(e1), "cuda")
    e2e = {"value": job_tops(world, dense_step, ems / ke), "unit": "TOPS", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": ke, "ms_per_step": ems / ke,
           "path": "pinned host X_t -> device, dstar_fmdq_linear per layer, Y_t -> pinned host; copies on "
                   "their own streams overlap the neighbouring steps' compute"}

    st = nat.status(sets[0][0].ws)
    for row in sets:
        for lay in row:
            st |= nat.status(lay.ws)
    if st:
        raise RuntimeError(f"device status {st} after the benchmark")

    if rank != 0:
        return

    # roofline of the dominant kernel, from the live event times
    peaks, peak_src = load_peaks()
    hbm = peaks["hbm_gbs"]
    i8_burst = peaks["bf16_tflops"] * INT8_PER_BF16
    kern = []
    for li, stt in enumerate(stats):
        kern.append(dict(kernel="quantize", layer=inputs[li].spec.name, ms=k1_ms[li], bound="hbm",
                         achieved=stt["k1_bytes"] / (k1_ms[li] * 1e-3) / 1e9, peak=hbm, unit="GB/s",
                         algorithmic=stt["k1_bytes"]))
        t_tc = stt["k2_issued"] / (i8_burst * 1e12)
        t_hbm = stt["k2_bytes"] / (hbm * 1e9)
        if t_tc >= t_hbm:
            kern.append(dict(kernel="slice_gemm", layer=inputs[li].spec.name, ms=k2_ms[li], bound="tensor",
                             achieved=stt["k2_dense"] / (k2_ms[li] * 1e-3) / 1e12, peak=i8_burst, unit="TOPS",
                             algorithmic=stt["k2_dense"]))
        else:
            kern.append(dict(kernel="slice_gemm", layer=inputs[li].spec.name, ms=k2_ms[li], bound="hbm",
                             achieved=stt["k2_bytes"] / (k2_ms[li] * 1e-3) / 1e9, peak=hbm, unit="GB/s",
                             algorithmic=stt["k2_bytes"]))
    for k in kern:
        k["frac"] = k["achieved"] / k["peak"]
    dom = max(kern, key=lambda k: k["ms"])
    traffic = load_traffic().get(f"{dom['kernel']}.{dom['layer']}.dram_bytes")
    roofline = {"bound": dom["bound"], "achieved": dom["achieved"], "peak": dom["peak"], "unit": dom["unit"],
                "frac": dom["frac"], "traffic": traffic, "kernel": f"{dom['kernel']} ({dom['layer']})",
                "peak_source": (f"{peak_src} hbm_gbs" if dom["bound"] == "hbm" else
                                f"{peak_src} bf16_tflops x {INT8_PER_BF16} (nominal int8:bf16)")}
    kernels = [{k: (round(v, 4) if isinstance(v, float) else v) for k, v in kk.items()} for kk in kern]

    cpu = None
    if not args.no_cpu_baseline:
        ops, el, desc, threads = oracle_sample_time(inputs, args.cpu_seconds)
        cpu = {"value": ops / el / 1e12, "unit": "TOPS", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": el}

    set_mb = sum(t.numel() * t.element_size() for lay in sets[0]
                 for t in (lay.x_a, lay.x_b, lay.x_prev, lay.y_prev, lay.w_q, lay.w_scale, lay.ws.buf)
                 if t is not None) / 1e6
    launches_per_step = 2 * nlayers  # quantizer and slice GEMM (slice-stream tiles run inside it) per layer
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": dict(workload_config(args.config, inputs, world, args.xprev),
                       l2=f"inputs rotate over {args.sets} buffer sets of {set_mb:.0f} MB each "
                          f"({args.sets * set_mb:.0f} MB > 126 MB L2); no flush needed"),
        "roofline": roofline,
        "kernels": kernels,
        "quantizer_GBps": [k["achieved"] for k in kern if k["kernel"] == "quantize"],
        "quantizer_frac_of_8TBs_spec": [k["achieved"] / 8000.0 for k in kern if k["kernel"] == "quantize"],
        "workload_stats": [{k: v for k, v in s.items() if k in ("bits_avg", "bit_hist", "planes_hist",
                                                              "fallback_tiles", "slice_macs")} for s in stats],
        "slice_macs_per_s": sum(s["slice_macs"] for s in stats) / (ms_step * 1e-3),
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * K,
        "clocks": clocks.summary(t_wall0, t_wall1),
        "kernel_sources": kernel_source_sha(),
        "timing": ("value: CUDA-graph replays of the captured dstar_fmdq_linear calls, one graph per cycle of "
                   f"{2 * args.sets} steps (every input set with both X_t); per-kernel times: a second timed "
                   "region of the step split into dstar_fmdq_quantize + dstar_fmdq_slice_gemm with event nodes "
                   "between the kernels" if graphs
                   else "eager C-ABI calls with CUDA events per kernel"),
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
