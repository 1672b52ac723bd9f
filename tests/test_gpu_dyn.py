"""GPU parity of FMDQ-DYN, the dynamic base (DSTAR section 3.1: the base of
Eqs. 2-3 is the minimum of M_i over all sub-channels, found by a first pass;
section 5.2, Table 2, DS-FMDQ-DYN) against the oracle's dynamic-base path:
the base itself, codes, widths, relative FPoT, g_ref, the encoded stream and
the int64 accumulators bit-exact; Y_t within the tolerance (bit-exact in
practice).  Through the C ABI with DSTAR_FLAG_DYNAMIC_BASE.
"""
import numpy as np
import pytest
import torch

from differential_quantized_gemm_b200 import _native as nat
from differential_quantized_gemm_b200 import synth

from gpu_helpers import dyn_parity, run_gpu, run_oracle_dyn, assert_quant_parity, assert_y_close

pytestmark = pytest.mark.gpu

SMALL_M = 3 * 128 + 48


@pytest.fixture(scope="module", autouse=True)
def _build():
    from differential_quantized_gemm_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


@pytest.mark.parametrize("cfg,layer", [(1, 0), (2, 0), (2, 1), (3, 0), (4, 1)], ids=lambda v: str(v))
def test_dyn_small(cfg, layer):
    M = 256 if cfg == 1 else (4096 if cfg == 4 else SMALL_M)
    inp = synth.make_layer(cfg, layer, M=M)
    g, q, acc, y, exact = dyn_parity(inp)
    assert exact > 0.999
    assert (q.pot >= 0).all() and (q.pot == 0).any()  # the minimum's own sub-channel has PoT 0


def test_dyn_adversarial_wide_spread():
    """Magnitudes over 2^24 in one batch: large PoTs, mixed widths, two-plane
    and slice-stream tiles."""
    inp = synth.adversarial_layer(SMALL_M, 1152, 512, seed=31, spread=24)
    g, q, acc, y, _ = dyn_parity(inp)
    assert (g["planes"] > 1).any()


@pytest.mark.parametrize("layer", [0, 1], ids=["ffn_up", "ffn_down"])
def test_dyn_full_size(layer):
    """The Latte video FFN at 16384 tokens, compared in full."""
    dyn_parity(synth.make_layer(4, layer))


def test_dyn_forced_8bit():
    inp = synth.make_layer(5, 0, step=10, force_bits=8, M=SMALL_M)
    g, q, acc, y, _ = dyn_parity(inp)
    assert (g["bits"] == 8).all()


def test_dyn_stage_split_equals_linear():
    """dstar_fmdq_quantize + dstar_fmdq_slice_gemm with the flag give the fused call's result."""
    inp = synth.make_layer(2, 0, M=256)
    a = run_gpu(inp, flags=nat.FLAG_DYNAMIC_BASE)
    from gpu_helpers import to_dev
    d = to_dev(inp)
    ws = nat.Workspace(inp.spec.M, inp.spec.K)
    base = 2.0 ** inp.spec.lb
    nat.quantize(d["x_t"], d["x_prev"], base, ws, flags=nat.FLAG_DYNAMIC_BASE)
    nat.slice_gemm(d["w_q"], d["w_scale"], d["y_prev"], base, ws, flags=nat.FLAG_DYNAMIC_BASE)
    torch.cuda.synchronize()
    assert nat.status(ws) == 0
    assert np.array_equal(d["y_prev"].float().cpu().numpy(), a["y"])


def test_dyn_stationary_keeps_output():
    inp = synth.make_layer(2, 0, M=128)
    inp.x_t = inp.x_prev.copy()
    g = run_gpu(inp, flags=nat.FLAG_DYNAMIC_BASE)
    assert g["status"] == 0
    base_bits = g["ws"].sections(128, inp.spec.K)["dyn_base"].cpu().view(torch.int32).item()
    assert base_bits == -1  # no nonzero M_i: the word keeps all bits set
    assert not g["codes"].any() and not g["acc"].any()
    assert np.array_equal(g["y"], inp.as_f32("y_prev"))
