"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
five synthetic workloads, at sizes the oracle finishes in seconds (several
128-row blocks plus a ragged tail) and at the full sizes, compared in full:
every code, bit width, FPoT, g_ref, record and int64 accumulator of every
tile, and Y_t element by element, both with the debug dumps and in the
launch the benchmark times (graph replay, y_out = y_prev, x_prev refreshed,
no debug buffers).
"""
import numpy as np
import pytest
import torch

import oracle
from differential_quantized_gemm_b200 import synth

from gpu_helpers import (assert_quant_parity, assert_y_close, full_parity, run_gpu, run_gpu_bench_launch,
                         run_oracle)

pytestmark = pytest.mark.gpu

SMALL_M = 3 * 128 + 48  # three full 128-row blocks and a ragged one (27 tiles)


@pytest.fixture(scope="module", autouse=True)
def _build():
    from differential_quantized_gemm_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _cases():
    for cfg in (1, 2, 3, 4):
        for li, spec in enumerate(synth.config_layers(cfg)):
            yield pytest.param(cfg, li, id=f"cfg{cfg}-{spec.name}")


@pytest.mark.parametrize("cfg,layer", list(_cases()))
def test_small_parity(cfg, layer):
    M = 256 if cfg == 1 else (4096 if cfg == 4 else SMALL_M)
    inp = synth.make_layer(cfg, layer, M=M)
    g, q, acc, y, exact = full_parity(inp)
    # cache refresh: x_prev now holds X_t, y_prev holds Y_t
    xt = torch.from_numpy(inp.x_t)
    xp_after = g["x_prev_after"].cpu()
    if inp.spec.dtype == "bf16":
        xp_after = xp_after.view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(xp_after, inp.x_t)
    else:
        assert np.array_equal(xp_after.numpy(), xt.numpy())
    assert exact > 0.999


FULL_CASES = [(2, 0), (2, 1), (3, 0), (3, 1), (3, 2), (3, 3), (4, 0), (4, 1)]


@pytest.mark.parametrize("cfg,layer", FULL_CASES, ids=lambda v: str(v))
def test_full_size_compared_in_full(cfg, layer):
    """Full-size workload, compared in full against one oracle run:
    (a) the benchmark's own launch (graph replay, Y in place, x_prev refreshed,
        no debug buffers): Y_t element by element and every integer section;
    (b) the same call with the debug dumps: every code and every int64
        accumulator of every tile."""
    inp = synth.make_layer(cfg, layer)
    q, acc, y = run_oracle(inp)
    b = run_gpu_bench_launch(inp)
    assert b["status"] == 0
    assert_quant_parity(b, q)
    assert_y_close(b["y"], y)
    xp = b["x_prev_after"].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(xp, inp.x_t), "x_prev refresh"
    g = run_gpu(inp)
    assert g["status"] == 0
    assert_quant_parity(g, q)
    assert np.array_equal(g["acc"], acc), "accumulators differ"
    assert np.array_equal(g["y"], b["y"]), "debug dumps changed Y_t"
    assert (g["planes"] <= 2).any()


def _chain_parity(chain):
    """Consecutive calls of one layer with caches carried on both sides
    independently (the oracle chains its own outputs); everything compared."""
    d = ws = yo = None
    for inp in chain.steps():
        if d is None:
            g = run_gpu(inp)
            d, ws = g["dev"], g["ws"]
        else:  # the device caches carry over: only X_t changes
            d["x_t"] = torch.from_numpy(inp.x_t).view(torch.bfloat16).cuda()
            g = run_gpu(inp, dev_bufs=d, ws=ws)
        q, acc, y = run_oracle(inp, y_prev_f32=yo)
        assert g["status"] == 0
        assert_quant_parity(g, q)
        assert np.array_equal(g["acc"], acc), "accumulators differ"
        assert_y_close(g["y"], y)
        yo = y
    return g, q


def test_sweep_chain_small():
    for layer in (0, 1):
        _chain_parity(synth.sweep_chain(layer, steps=[0, 1, 2, 24, 25, 49], M=512))


# first and last layer of the 28-layer stack, both projections of each
SWEEP_LAYERS = [(0, "l0_up"), (1, "l0_down"), (54, "l27_up"), (55, "l27_down")]


@pytest.mark.parametrize("layer", [li for li, _ in SWEEP_LAYERS], ids=[n for _, n in SWEEP_LAYERS])
def test_sweep_full_size(layer):
    """The timestep sweep at its full size (8192 tokens): steps 0, 1, 24, 25
    and 49 of the U-shaped schedule in a row, caches carried."""
    _chain_parity(synth.sweep_chain(layer, steps=[0, 1, 24, 25, 49], M=8192))


@pytest.mark.parametrize("force", [2, 8])
def test_forced_extremes_small(force):
    inp = synth.make_layer(5, 0, step=10, force_bits=force, M=SMALL_M)
    g, q, acc, y, _ = full_parity(inp)
    assert (g["bits"] == force).all()


@pytest.mark.parametrize("force", [2, 8])
@pytest.mark.parametrize("layer", [0, 1], ids=["up", "down"])
def test_forced_extremes_full_size(force, layer):
    """The all-2-bit and all-8-bit runs of the sweep at 8192 tokens, compared in full."""
    inp = synth.make_layer(5, layer, step=10, force_bits=force)
    g, q, acc, y, _ = full_parity(inp)
    assert (g["bits"] == force).all()
    if force == 8:
        assert (g["planes"] > 1).any(), "8-bit tiles should need more than one operand plane"


def test_adversarial_uses_slice_stream_for_wide_tiles():
    """Tiles whose shift-folded operands need more than two int8 planes go
    through the slice-stream kernel; results stay bit-exact."""
    inp = synth.adversarial_layer(SMALL_M, 1152, 512, seed=21, spread=30)
    g, q, acc, y, _ = full_parity(inp)
    assert (g["planes"] > 2).any() and (g["planes"] <= 2).any()


def test_two_plane_tiles():
    inp = synth.adversarial_layer(SMALL_M, 1152, 512, seed=22, spread=12)
    g, q, acc, y, _ = full_parity(inp)
    assert (g["planes"] == 2).any()


def test_slice_path_flag_matches_tensor_cores():
    from differential_quantized_gemm_b200 import FLAG_SLICE_PATH
    inp = synth.make_layer(2, 0, M=256)
    a = run_gpu(inp)
    b = run_gpu(inp, flags=FLAG_SLICE_PATH)
    assert np.array_equal(a["acc"], b["acc"])
    assert np.array_equal(a["y"], b["y"])
    q, acc, y = run_oracle(inp)
    assert np.array_equal(b["acc"], acc)
