"""Host-side formulas of the benchmark: the algorithmic byte and op counts the
roofline fractions divide by, and the workload description both arms print."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from differential_quantized_gemm_b200 import synth  # noqa: E402


def _sections(T, K, counts, planes, mask_words=1, masks=None):
    return {"count": torch.tensor(counts, dtype=torch.int32),
            "planes": torch.tensor(planes, dtype=torch.int32),
            "mask1": torch.tensor(np.asarray(masks if masks is not None else np.zeros((T, mask_words)),
                                             dtype=np.uint32).view(np.int32))}


def test_k1_bytes_by_hand():
    spec = synth.LayerSpec("t", 32, 64, 16, "bf16", -4, 0, 0)
    sec = _sections(2, 64, [40, 8], [1, 2])
    M, K = 32, 64
    # X_t, X_{t-1} read + X_{t-1} refresh (2 B each), plane 0 (1 B), plane 1 for the
    # 16 rows of the two-plane tile, 8 B per record, FPoT and width per sub-channel
    expect = 3 * M * K * 2 + M * K + 16 * K + 48 * 8 + 2 * 2 * K
    assert bench.algorithmic_k1_bytes(spec, sec) == expect
    # with two resident buffers there is no refresh write
    assert bench.algorithmic_k1_bytes(spec, sec, refresh=False) == expect - M * K * 2


def test_k2_ops_and_bytes_by_hand():
    spec = synth.LayerSpec("t", 256, 256, 128, "bf16", -4, 0, 0)
    # two 128-row blocks; the second needs plane 1 on K chunks 0 and 1 (one tile's mask)
    masks = np.zeros((16, 1), np.uint32)
    masks[9, 0] = 0b11
    sec = _sections(16, 256, [0] * 16, [1] * 8 + [2] * 8, masks=masks)
    dense, issued, byts, nfall = bench.algorithmic_k2(spec, sec)
    M, K, N = 256, 256, 128
    assert dense == 2.0 * M * N * K
    assert issued == dense + 2 * (2.0 * 128 * N * 128)
    assert byts == 2 * M * N * 2 + N * K + M * K + 2 * 128 * 128
    assert nfall == 0


def test_workload_config_names_the_xprev_mode():
    inputs = bench.workload_inputs(1, 0)
    a = bench.workload_config(1, inputs, 1)
    b = bench.workload_config(1, inputs, 1, "swap")
    assert a["x_prev"] == bench.XPREV_DESC["copy"] and b["x_prev"] == bench.XPREV_DESC["swap"]
    assert {k: v for k, v in a.items() if k != "x_prev"} == {k: v for k, v in b.items() if k != "x_prev"}


def test_job_throughput_counts_every_rank():
    assert bench.job_tops(4, 1e12, 1.0) == 4 * bench.job_tops(1, 1e12, 1.0)


def test_oracle_baseline_reports_stages_threads_and_cpu():
    """The CPU baseline: all threads with a per-stage split, one thread on a
    small sample, and the CPU model."""
    inputs = bench.workload_inputs(1, 0)
    cpu = bench.oracle_baseline(inputs, 0.2)
    assert cpu["kind"] == "oracle" and cpu["value"] > 0 and cpu["cores"] >= 1
    assert set(cpu["stages_s"]) == {"quantize", "gemm", "epilogue"}
    assert cpu["single_thread"]["cores"] == 1 and cpu["single_thread"]["value"] > 0
    assert isinstance(cpu["cpu_model"], str) and cpu["cpu_model"]
    import oracle
    assert oracle.n_threads() == os.cpu_count() or oracle.n_threads() >= 1  # restored after the 1-thread run


def test_bench_defaults_to_the_largest_workload():
    args = bench.parse([])
    assert args.config == 4 and args.steps > 0 and args.warmup >= 3
    from differential_quantized_gemm_b200 import synth
    assert max(s.M for s in synth.config_layers(args.config)) == 16384
