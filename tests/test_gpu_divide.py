"""The division by the dynamic base (FMDQ-DYN, DSTAR section 3.1 step 1: the
codes of fl32(dX / base)) against CUDA's __fdiv_rn, bit for bit, on the GPU
(dstar_fmdq_selftest_div): every significand of the dividend in five binades
for divisors with random significands across the range the FMA path serves,
divisors whose significands are all ones, 1, 1 + 2^-23 and 1.5, the range's
end points, and divisors outside it (which take the IEEE division)."""
import numpy as np
import pytest
import torch

from differential_quantized_gemm_b200 import _native as nat

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from differential_quantized_gemm_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _divisors():
    rng = np.random.default_rng(7)
    sig = rng.integers(0, 1 << 23, 48, dtype=np.uint32)
    exp = rng.integers(-100, 100, 48)
    b = [np.uint32(((e + 127) << 23) | s).view(np.float32) for s, e in zip(sig, exp)]
    for e in (-100, -37, -1, 0, 1, 29, 99):
        for s in ((1 << 23) - 1, 0, 1, 1 << 22):  # all-ones, 1, 1 + 2^-23, 1.5
            b.append(np.uint32(((e + 127) << 23) | s).view(np.float32))
    b += [np.float32(2.0 ** 100), np.float32(-3.5), np.float32(-(2.0 ** -100))]
    return torch.tensor(np.array(b, dtype=np.float32), device="cuda")


def test_dynamic_base_division_equals_ieee_division():
    b = _divisors()
    assert nat.selftest_div(b, -20, -18) == 0
    assert nat.selftest_div(b, -1, 1) == 0
    assert nat.selftest_div(b, 19, 21) == 0


def test_divisors_outside_the_fast_range_use_ieee_division():
    b = torch.tensor([2.0 ** -110, 2.0 ** 110, 1e-40, -(2.0 ** 120)], dtype=torch.float32, device="cuda")
    assert nat.selftest_div(b, -3, 3) == 0


def test_selftest_rejects_bad_arguments():
    b = torch.ones(1, device="cuda")
    with pytest.raises(nat.DstarError):
        nat.selftest_div(b, -127, 0)
