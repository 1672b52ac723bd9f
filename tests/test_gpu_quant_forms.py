"""The quantizer's launch forms at their boundaries, each compared with the
oracle in full (DSTAR section 3.1 steps 1-4; codes, FPoT, widths, records,
planes, accumulators and Y_t):

- one tile per cluster of CTAs for batches of fewer than two tiles per SM,
  and for every batch whose double buffers do not fit an SM (K = DSTAR_K_MAX);
- the persistent kernel with two CTAs of 4 + 4 warps per SM (at most four
  tiles per SM and two CTAs' buffers in the SM's shared memory);
- the persistent kernel with one CTA of 8 + 8 warps per SM (more tiles per
  SM, or channels whose buffers fit only once)."""
import pytest
import torch

from differential_quantized_gemm_b200 import _native as nat
from differential_quantized_gemm_b200 import synth

from gpu_helpers import full_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from differential_quantized_gemm_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("tiles_per_sm,K,N", [
    (2, nat.K_MAX, 48),  # buffers too large for the persistent kernel: clusters over the channels
    (4, 1152, 48),       # the last batch of two CTAs per SM
    (4.25, 1152, 48),    # past four tiles per SM: one CTA per SM
    (2, 2848, 32),       # two CTAs' buffers still fit an SM
    (2, 2880, 32),       # they no longer do
])
def test_quantizer_form_boundaries(tiles_per_sm, K, N):
    M = 16 * int(round(tiles_per_sm * _sms()))
    inp = synth.adversarial_layer(M, K, N, seed=int(7 * tiles_per_sm + K), spread=12)
    full_parity(inp)
