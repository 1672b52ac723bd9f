"""Host logic of the multi-rank benchmark path, on CPU with `gloo` ranks.

The batch split needs no data exchange: each rank runs its own batch of the
same workload, and the only collectives are the barrier around the timed region
and the max of the ranks' times.  These tests run two processes and check
that reduction, the whole-job throughput formula, the per-rank inputs (same
shapes, different draws), that the reference arm does nothing off rank 0, and
that splitting one batch by token tiles across two ranks reproduces the whole
batch's accumulators and Y_t bit for bit (the oracle on each half).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as td
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    td.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # the slowest rank's time is the job's time
        t = bench.max_over_ranks(1.5 + rank, "cpu")
        # per-rank inputs: identical shapes, independent draws
        inp = bench.workload_inputs(1, rank)
        gathered = [None] * world
        td.all_gather_object(gathered, (inp[0].spec.M, inp[0].spec.K, inp[0].spec.N, float(inp[0].x_t[0, 0])))
        # the reference arm runs on rank 0 only; other ranks return at once
        ref = None
        if rank != 0:
            class A:
                config = 1
                steps = 1
                warmup = 3
            ref = bench.run_reference(A(), rank, world)
        # the batch split itself: each rank runs the oracle on its own whole
        # 16-token tiles of one batch; together they must give the whole
        # batch's Y_t (rows of Y depend only on the same rows of dX)
        import oracle
        from differential_quantized_gemm_b200 import synth
        whole = synth.make_layer(2, 0, M=256)
        T = whole.spec.M // 16
        lo, hi = 16 * (T * rank // world), 16 * (T * (rank + 1) // world)
        rows = slice(lo, hi)
        _, acc, y = oracle.linear(whole.as_f32("x_t")[rows], whole.as_f32("x_prev")[rows],
                                  whole.as_f32("y_prev")[rows], whole.w_q, whole.w_scale, whole.spec.lb)
        parts = [None] * world
        td.all_gather_object(parts, (lo, hi, acc, y))
        td.barrier()
        out[rank] = (t, gathered, ref, parts if rank == 0 else None)
    finally:
        td.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], codes
    for r in range(world):
        t, gathered, ref, _ = res[r]
        assert t == pytest.approx(2.5)
        assert gathered[0][:3] == gathered[1][:3]
        assert gathered[0][3] != gathered[1][3]
        assert ref is None
    # the shards, stacked in rank order, are the whole batch's result bit for bit
    import oracle
    from differential_quantized_gemm_b200 import synth
    parts = res[0][3]
    whole = synth.make_layer(2, 0, M=256)
    _, acc, y = oracle.linear(whole.as_f32("x_t"), whole.as_f32("x_prev"), whole.as_f32("y_prev"), whole.w_q,
                              whole.w_scale, whole.spec.lb)
    assert [p[0] for p in parts] == [0, 128] and [p[1] for p in parts] == [128, 256]
    assert np.array_equal(np.concatenate([p[2] for p in parts]), acc)
    assert np.array_equal(np.concatenate([p[3] for p in parts]), y)


def test_job_throughput_is_weak_scaling():
    ops = 2.0 * 2048 * 4608 * 1152 * 2
    one = bench.job_tops(1, ops, 0.1)
    assert one == pytest.approx(ops / 1e-4 / 1e12)
    assert bench.job_tops(4, ops, 0.1) == pytest.approx(4 * one)
    # single process: the reduction is the identity
    assert bench.max_over_ranks(3.25) == 3.25
    assert np.isfinite(one)
