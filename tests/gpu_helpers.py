"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
the CPU oracle on the same seeded inputs, and compare them.

Bar (fixed before any kernel ran): codes, bit widths, FPoT, g_ref, record
counts, the encoded stream and the accumulators bit-exact; Y_t within
max-abs 1e-2 and relative L2 1e-3 of the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from differential_quantized_gemm_b200 import _native as nat
from differential_quantized_gemm_b200 import synth

Y_MAX_ABS = 1e-2
Y_REL_L2 = 1e-3


def to_dev(inp: synth.LayerInputs, dev="cuda"):
    def f(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if inp.spec.dtype == "bf16":
            t = t.view(torch.bfloat16)
        return t.to(dev)

    return dict(x_t=f(inp.x_t), x_prev=f(inp.x_prev), y_prev=f(inp.y_prev),
                w_q=torch.from_numpy(inp.w_q).to(dev), w_scale=torch.from_numpy(inp.w_scale).to(dev))


def dev_to_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def run_gpu(inp: synth.LayerInputs, t0=None, force_bits=None, flags=0, y_distinct=False, debug=True,
            ws: nat.Workspace | None = None, dev_bufs=None):
    spec = inp.spec
    M, K, N = spec.M, spec.K, spec.N
    d = to_dev(inp) if dev_bufs is None else dev_bufs
    if ws is None:
        ws = nat.Workspace(M, K)
    codes = torch.zeros(M, K, dtype=torch.int8, device="cuda") if debug else None
    acc = torch.zeros(M, N, dtype=torch.int64, device="cuda") if debug else None
    y_out = torch.empty_like(d["y_prev"]) if y_distinct else None
    out = nat.linear(d["x_t"], d["x_prev"], d["y_prev"], d["w_q"], d["w_scale"], 2.0 ** spec.lb, ws,
                     t0=spec.t0 if t0 is None else t0, force_bits=spec.force_bits if force_bits is None else force_bits,
                     flags=flags, y_out=y_out, debug_codes=codes, debug_acc=acc)
    torch.cuda.synchronize()
    st = nat.status(ws)
    sec = ws.sections(M, K)
    res = dict(status=st, y=dev_to_f32(out), x_prev_after=d["x_prev"], y_prev_after=d["y_prev"],
               fpot=sec["fpot"].cpu().numpy(), bits=sec["bits"].cpu().numpy(), g_ref=sec["g_ref"].cpu().numpy(),
               count=sec["count"].cpu().numpy(), planes=sec["planes"].cpu().numpy(),
               records=sec["records"].cpu().numpy().view(np.uint32), dev=d, ws=ws)
    if debug:
        res["codes"] = codes.cpu().numpy()
        res["acc"] = acc.cpu().numpy()
    return res


def run_gpu_bench_launch(inp: synth.LayerInputs):
    """The call exactly as the benchmark times it: dstar_fmdq_linear captured in
    a CUDA graph and replayed, y_out = y_prev (in place), x_prev refreshed, no
    debug buffers.  Returns Y_t, the refreshed caches and the workspace's
    integer sections."""
    spec = inp.spec
    d = to_dev(inp)
    ws = nat.Workspace(spec.M, spec.K)
    x_t_live = d["x_t"].clone()  # the graph reads this buffer; the inputs are copied into it before replay
    x_prev_live = torch.empty_like(d["x_prev"])
    y_live = torch.empty_like(d["y_prev"])
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=side):
        nat.linear(x_t_live, x_prev_live, y_live, d["w_q"], d["w_scale"], 2.0 ** spec.lb, ws, t0=spec.t0,
                   force_bits=spec.force_bits)
    x_prev_live.copy_(d["x_prev"])
    y_live.copy_(d["y_prev"])
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    st = nat.status(ws)
    sec = ws.sections(spec.M, spec.K)
    res = dict(status=st, y=dev_to_f32(y_live), x_prev_after=x_prev_live,
               fpot=sec["fpot"].cpu().numpy(), bits=sec["bits"].cpu().numpy(), g_ref=sec["g_ref"].cpu().numpy(),
               count=sec["count"].cpu().numpy(), planes=sec["planes"].cpu().numpy(),
               records=sec["records"].cpu().numpy().view(np.uint32))
    del g
    return res


def run_oracle(inp: synth.LayerInputs, t0=None, force_bits=None, tiles=None, y_prev_f32=None):
    spec = inp.spec
    q = oracle.quantize(inp.as_f32("x_t"), inp.as_f32("x_prev"), spec.lb, spec.t0 if t0 is None else t0,
                        spec.force_bits if force_bits is None else force_bits)
    acc = oracle.acc_direct(q, inp.w_q, tiles)
    yp = inp.as_f32("y_prev") if y_prev_f32 is None else y_prev_f32
    y = oracle.epilogue_f32(acc, q.g_ref, spec.lb, inp.w_scale, yp, spec.dtype == "bf16", tiles)
    return q, acc, y


def tile_rows(T, tiles):
    if tiles is None:
        return slice(None)
    return np.concatenate([np.arange(16 * t, 16 * t + 16) for t in tiles])


def assert_quant_parity(g, q):
    """Every integer output of the quantizer; the codes only when they were dumped."""
    if "codes" in g:
        assert np.array_equal(g["codes"], q.codes), "codes differ"
    assert np.array_equal(g["bits"], q.bits), "bit widths differ"
    assert np.array_equal(g["fpot"], q.fpot), "FPoT differs"
    assert np.array_equal(g["g_ref"], q.g_ref), "g_ref differs"
    assert np.array_equal(g["count"], q.count), "record counts differ"
    rec = g["records"]  # [T, cap, 2] uint32
    cap = q.cap
    live = np.arange(cap)[None, :] < q.count[:, None]
    word = rec[:, :, 0]
    meta = rec[:, :, 1]
    k = (meta & 0xFFFF).astype(np.uint16)
    tag = ((meta >> 16) & 0xFF).astype(np.uint8).view(np.int8)
    j = (meta >> 24).astype(np.uint8)
    assert np.array_equal(word[live], q.rec_word[live]), "slice words differ"
    assert np.array_equal(k[live], q.rec_k[live]), "record channels differ"
    assert np.array_equal(tag[live], q.rec_tag[live]), "record FPoT tags differ"
    assert np.array_equal(j[live], q.rec_j[live]), "record slice indices differ"


def y_errors(y_gpu, y_orc):
    diff = np.abs(y_gpu.astype(np.float64) - y_orc.astype(np.float64))
    max_abs = float(diff.max()) if diff.size else 0.0
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(y_orc.astype(np.float64)), 1e-30))
    exact = float((y_gpu == y_orc).mean()) if diff.size else 1.0
    return max_abs, rel, exact


def assert_y_close(y_gpu, y_orc):
    max_abs, rel, exact = y_errors(y_gpu, y_orc)
    assert max_abs <= Y_MAX_ABS and rel <= Y_REL_L2, (max_abs, rel, exact)
    return exact


def full_parity(inp, tiles=None, flags=0, y_distinct=False, t0=None, force_bits=None):
    """Run both sides and compare everything; tiles restricts the accumulator/Y comparison."""
    g = run_gpu(inp, t0=t0, force_bits=force_bits, flags=flags, y_distinct=y_distinct)
    q, acc, y = run_oracle(inp, t0=t0, force_bits=force_bits, tiles=tiles)
    assert g["status"] == 0, g["status"]
    assert_quant_parity(g, q)
    rows = tile_rows(q.T, tiles)
    assert np.array_equal(g["acc"][rows], acc[rows]), "accumulators differ"
    exact = assert_y_close(g["y"][rows], y[rows])
    return g, q, acc, y, exact


def run_oracle_dyn(inp: synth.LayerInputs, y_prev_f32=None):
    """The oracle with the dynamic base; the call's base_scale (2^lb) sets the thresholds."""
    spec = inp.spec
    q = oracle.quantize_dyn(inp.as_f32("x_t"), inp.as_f32("x_prev"), spec.lb, spec.t0, spec.force_bits)
    acc = oracle.acc_direct(q, inp.w_q)
    yp = inp.as_f32("y_prev") if y_prev_f32 is None else y_prev_f32
    y = oracle.epilogue_dyn_f32(acc, q.g_ref, q.base, inp.w_scale, yp, spec.dtype == "bf16")
    return q, acc, y


def dyn_parity(inp, debug=True, flags=0):
    """Dynamic base: GPU (DSTAR_FLAG_DYNAMIC_BASE, plus `flags`) against the oracle, everything compared."""
    g = run_gpu(inp, flags=nat.FLAG_DYNAMIC_BASE | flags, debug=debug)
    q, acc, y = run_oracle_dyn(inp)
    assert g["status"] == 0, g["status"]
    base = float(g["ws"].sections(inp.spec.M, inp.spec.K)["dyn_base"].cpu()[0])
    assert base == q.base, (base, q.base)
    assert_quant_parity(g, q)
    if debug:
        assert np.array_equal(g["acc"], acc), "accumulators differ"
    exact = assert_y_close(g["y"], y)
    return g, q, acc, y, exact
