"""GPU parity of every output tile form of the slice GEMM (DSTAR section 3.1
step 5, section 4.2 "Design of MPU"): 128 x 128 and 128 x 256 in one CTA,
and 256 x 256 / 256 x 128 in a cluster of two CTAs whose tensor-core
instructions span both SMs (each holds 128 rows of the operand plane and half
of the weight tile).  Each form is
forced through the call's tile flag on ragged shapes -- a last tile whose
second half is partly or wholly beyond M, output columns that end inside a
tile -- with two-plane tiles and tiles left to the slice stream, and compared
with the oracle in full (every code and accumulator, Y_t within the bar).
The forms give the same accumulators bit for bit."""
import numpy as np
import pytest
import torch

from differential_quantized_gemm_b200 import _native as nat
from differential_quantized_gemm_b200 import synth

from gpu_helpers import assert_quant_parity, assert_y_close, full_parity, run_gpu_bench_launch, run_oracle

pytestmark = pytest.mark.gpu

FORMS = [nat.TILE_128x128, nat.TILE_128x256, nat.TILE_PAIR_256x256, nat.TILE_PAIR_256x128]


@pytest.fixture(scope="module", autouse=True)
def _build():
    from differential_quantized_gemm_b200 import build
    build.build()
    assert torch.cuda.is_available()


def test_tile_shapes_of_the_workloads():
    # the Latte FFN pair: CTA pairs of 256 x 256 for the up-projection (every
    # SM's 128 x 256 epilogue bounds it, with half the weight bytes per SM of
    # a one-CTA tile), pairs of 256 x 128 for the down-projection (K = 4608)
    assert nat.gemm_tile(16384, 4608, 1152, True) == (256, 256, True)
    assert nat.gemm_tile(16384, 1152, 4608, True) == (256, 128, True)
    valid = {(128, 128, False), (128, 256, False), (256, 256, True), (256, 128, True)}
    for M, N, K in [(2048, 4608, 1152), (2048, 1152, 4608), (8192, 3456, 1152), (432, 1152, 1152), (16, 16, 32)]:
        assert nat.gemm_tile(M, N, K, True) in valid
        bm, bn, pair = nat.gemm_tile(M, N, K, False)
        assert bn == 128 and (bm, pair) in {(128, False), (256, True)}  # fp32 outputs: 128-column tiles


def test_unknown_tile_form_is_rejected():
    inp = synth.make_layer(2, 0, M=128)
    with pytest.raises(nat.DstarError, match="tile form"):
        full_parity(inp, flags=nat.tile_flag(7))


# M = 432: the last 256-row tile's second half is ragged; M = 3856: it lies
# wholly beyond M; N = 400 ends inside a 128- and a 256-column tile
@pytest.mark.parametrize("form", FORMS)
@pytest.mark.parametrize("M,N", [(432, 1152), (3856, 400)])
def test_form_two_plane_tiles(form, M, N):
    inp = synth.adversarial_layer(M, 1152, N, seed=40 + M % 7, spread=12)
    g, q, acc, y, _ = full_parity(inp, flags=nat.tile_flag(form))
    assert (g["planes"] == 2).any()


@pytest.mark.parametrize("form", FORMS)
def test_form_slice_stream_tiles(form):
    inp = synth.adversarial_layer(432, 1152, 512, seed=21, spread=30)
    g, q, acc, y, _ = full_parity(inp, flags=nat.tile_flag(form))
    assert (g["planes"] > 2).any() and (g["planes"] <= 2).any()


@pytest.mark.parametrize("form", [nat.TILE_128x128, nat.TILE_PAIR_256x128])
def test_form_fp32_outputs(form):
    inp = synth.adversarial_layer(400, 256, 272, seed=6, spread=8, dtype="f32")
    full_parity(inp, flags=nat.tile_flag(form))


def test_forms_give_identical_results():
    inp = synth.make_layer(3, 3, M=1024)  # the PixArt down-projection's shape at 1024 tokens
    ys = []
    for form in FORMS:
        g = full_parity(inp, flags=nat.tile_flag(form))[0]
        ys.append((g["acc"], g["y"]))
    for acc, y in ys[1:]:
        assert np.array_equal(acc, ys[0][0]) and np.array_equal(y, ys[0][1])


def test_library_choice_in_the_benchmark_launch():
    """Graph-replayed, in place, no debug buffers, the library's tile choice:
    Y_t against the oracle at the Latte down-projection's shape (4096 tokens)."""
    inp = synth.make_layer(4, 1, M=4096)
    g = run_gpu_bench_launch(inp)
    q, acc, y = run_oracle(inp)
    assert g["status"] == 0
    assert_quant_parity(g, q)
    assert_y_close(g["y"], y)
