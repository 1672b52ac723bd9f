"""Pins of the oracle's GELU (the activation fused between the two layers of a
DiT feed-forward block, DSTAR section 4.3 "Operator Mapping") and of the
chained pair: closed-form values, the identity GELU(y) - GELU(-y) = y,
element-wise agreement with Python's math.erf, bf16 rounding, and the chain
equal to its two linear calls with the GELU output between them.  CPU only.
"""
import math

import numpy as np

from differential_quantized_gemm_b200 import synth


def _gelu_math(v: float) -> float:
    return 0.5 * v * math.erfc(-v / math.sqrt(2.0))


def test_closed_form_values(orc):
    y = np.array([0.0, 1.0, -1.0, 3.0, -3.0, 8.0, -8.0], np.float32)
    g = orc.gelu(y, False)
    assert g[0] == 0.0
    assert g[1] == np.float32(0.8413447460685429)          # Phi(1)
    assert g[2] == np.float32(-0.15865525393145705)         # -1 * Phi(-1)
    assert g[5] == np.float32(8.0) and abs(g[6]) < 1e-14     # tails: y and 0


def test_odd_part_identity():
    """GELU(y) - GELU(-y) = y(Phi(y) + Phi(-y)) = y, up to fp32 rounding of each term."""
    import oracle
    y = np.random.default_rng(0).standard_normal(4096).astype(np.float32) * 3
    gp, gm = oracle.gelu(y, False).astype(np.float64), oracle.gelu(-y, False).astype(np.float64)
    err = np.abs(gp - gm - y.astype(np.float64))
    assert (err <= 2.0 ** -23 * (np.abs(gp) + np.abs(gm)) + 1e-30).all()


def test_against_math_erfc_elementwise(orc):
    y = np.concatenate([np.linspace(-12, 6, 3001), np.random.default_rng(1).standard_normal(2000) * 2]).astype(np.float32)
    g = orc.gelu(y, False)
    ref = np.array([np.float32(_gelu_math(float(v))) for v in y])
    assert np.array_equal(g, ref)
    gb = orc.gelu(y, True)
    assert np.array_equal(gb, orc.bf16_to_f32(orc.f32_to_bf16(ref)))
    # the erf form of the same function agrees where 1 + erf does not cancel
    mid = y > -2
    erf_form = np.array([np.float32(0.5 * float(v) * (1.0 + math.erf(float(v) / math.sqrt(2.0)))) for v in y[mid]])
    assert np.allclose(g[mid], erf_form, rtol=1e-6, atol=1e-12)
    # and the negative tail keeps its relative accuracy (no cancellation)
    assert g[0] < 0 and abs(g[0] / np.float32(-12 * 0.5 * math.erfc(12 / math.sqrt(2.0))) - 1) < 1e-6


def test_chain_is_two_linears_with_gelu_between(orc):
    up = synth.make_layer(2, 0, M=32)
    s = up.spec
    w2, ws2 = synth.layer_weights(2, 1)
    rng = np.random.default_rng(4)
    y1p = up.as_f32("y_prev")
    hp = orc.gelu(y1p, True)
    y2p = orc.bf16_to_f32(orc.f32_to_bf16(rng.standard_normal((32, w2.shape[0])).astype(np.float32)))
    out = orc.ffn_gelu(up.as_f32("x_t"), up.as_f32("x_prev"), y1p, up.w_q, up.w_scale, hp, y2p, w2, ws2, s.lb)
    q1, acc1, y1, h, q2, acc2, y2 = out
    _, a1, b1 = orc.linear(up.as_f32("x_t"), up.as_f32("x_prev"), y1p, up.w_q, up.w_scale, s.lb)
    assert np.array_equal(acc1, a1) and np.array_equal(y1, b1)
    assert np.array_equal(h, orc.gelu(y1, True))
    _, a2, b2 = orc.linear(h, hp, y2p, w2, ws2, s.lb)
    assert np.array_equal(acc2, a2) and np.array_equal(y2, b2)
    assert q2.codes.any()  # the second layer sees a nonzero differential
