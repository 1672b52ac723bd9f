"""Seeded random shapes through the whole call (DSTAR section 3.1, every step
of the FMDQ differential linear) against the oracle: M, K and N drawn within
the interface's rules (M % 16 == 0, K % 32 == 0, N % 16 == 0), bf16 or fp32,
a random slice-GEMM tile form (one CTA or a CTA pair), a random dX spread
(from one-plane tiles to the slice stream) and sometimes a distinct output;
then with the dynamic base (FMDQ-DYN).  Every code, tag, record and
accumulator bit-exact, Y_t within the bar."""
import numpy as np
import pytest
import torch

from differential_quantized_gemm_b200 import _native as nat
from differential_quantized_gemm_b200 import synth

from gpu_helpers import dyn_parity, full_parity

pytestmark = pytest.mark.gpu

FORMS = [0, nat.TILE_128x128, nat.TILE_128x256, nat.TILE_PAIR_256x256, nat.TILE_PAIR_256x128]


@pytest.fixture(scope="module", autouse=True)
def _build():
    from differential_quantized_gemm_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _case(i):
    rng = np.random.default_rng(1000 + i)
    M = 16 * int(rng.integers(1, 80))
    K = 32 * int(rng.integers(1, 72))
    N = 16 * int(rng.integers(1, 72))
    dtype = "bf16" if rng.random() < 0.75 else "f32"
    spread = int(rng.choice([4, 8, 12, 20, 30]))
    form = int(rng.choice(FORMS))
    distinct = bool(rng.random() < 0.3)
    return M, K, N, dtype, spread, form, distinct


@pytest.mark.parametrize("i", range(64))
def test_random_shape(i):
    M, K, N, dtype, spread, form, distinct = _case(i)
    inp = synth.adversarial_layer(M, K, N, seed=2000 + i, spread=spread, dtype=dtype)
    g, q, acc, y, _ = full_parity(inp, flags=nat.tile_flag(form), y_distinct=distinct)
    if distinct:
        assert np.array_equal(g["y_prev_after"].float().cpu().numpy(), g["y"])


@pytest.mark.parametrize("i", range(16))
def test_random_shape_dynamic_base(i):
    M, K, N, dtype, spread, form, _ = _case(100 + i)
    inp = synth.adversarial_layer(M, K, N, seed=3000 + i, spread=spread, dtype=dtype)
    dyn_parity(inp, flags=nat.tile_flag(form))
