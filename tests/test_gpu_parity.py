"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
five synthetic workloads, at sizes the oracle finishes in seconds (several
128-row blocks plus a ragged tail) and at the full sizes in the launch
configuration the benchmark times (y_out = y_prev, x_prev refreshed), with
accumulators and Y_t compared on sampled token tiles there.
"""
import numpy as np
import pytest
import torch

import oracle
from differential_quantized_gemm_b200 import synth

from gpu_helpers import assert_quant_parity, assert_y_close, full_parity, run_gpu, run_oracle, tile_rows

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


@pytest.mark.parametrize("cfg,layer", [(2, 0), (2, 1), (3, 0), (3, 1), (3, 2), (3, 3), (4, 0), (4, 1)],
                         ids=lambda v: str(v))
def test_full_size_sampled(cfg, layer):
    """Full-size workload in the benchmark's launch configuration; every integer
    stage compared in full, accumulators and Y_t on sampled tiles."""
    inp = synth.make_layer(cfg, layer)
    T = inp.spec.M // 16
    rng = np.random.default_rng(cfg * 10 + layer)
    tiles = np.unique(np.concatenate([[0, T - 1, T // 2], rng.choice(T, 13, replace=False)]))
    g = run_gpu(inp)
    q, acc, y = run_oracle(inp, tiles=tiles)
    assert g["status"] == 0
    assert_quant_parity(g, q)
    rows = tile_rows(T, tiles)
    assert np.array_equal(g["acc"][rows], acc[rows])
    assert_y_close(g["y"][rows], y[rows])
    assert (g["planes"] <= 2).any()


def test_sweep_chain_with_caches():
    """Timestep sweep: consecutive steps with caches carried on both sides
    independently (the oracle chains its own outputs)."""
    M = 512
    for layer in (0, 1):
        chain = synth.sweep_chain(layer, steps=[0, 1, 2, 24, 25, 49], M=M)
        spec = chain.spec
        d = None
        yo = None
        for inp in chain.steps():
            if d is None:
                g = run_gpu(inp)
                d = g["dev"]
                ws = g["ws"]
            else:
                # the device caches carry over: only X_t changes
                d["x_t"] = torch.from_numpy(inp.x_t).view(torch.bfloat16).cuda()
                g = run_gpu(inp, dev_bufs=d, ws=ws)
            q, acc, y = run_oracle(inp, y_prev_f32=yo)
            assert g["status"] == 0
            assert_quant_parity(g, q)
            assert np.array_equal(g["acc"], acc)
            assert_y_close(g["y"], y)
            yo = y
        assert spec.K in (1152, 4608)


@pytest.mark.parametrize("force", [2, 8])
def test_forced_extremes(force):
    inp = synth.make_layer(5, 0, step=10, force_bits=force, M=SMALL_M)
    g, q, acc, y, _ = full_parity(inp)
    assert (g["bits"] == force).all()


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
