"""Pins of the oracle's dynamic-base path (FMDQ-DYN): the base of Eqs. 2-3
taken as the minimum of M_i over the call's sub-channels (DSTAR section 3.1
"On-the-Fly PoT-Based Quantization"; the DS-FMDQ-DYN variant of section 5.2,
Table 2), checked against things other than the oracle itself: a brute-force
minimum, exact rational arithmetic (Python fractions) for PoT, widths and
codes, the reduction to the static quantizer when the minimum is a power of
two, the quantization error bound on tiny shapes, and the stationary case.
CPU only.
"""
from fractions import Fraction

import numpy as np
import pytest

from differential_quantized_gemm_b200 import synth


def _small(M=48, K=64):
    inp = synth.make_layer(2, 0, M=M)
    return inp.as_f32("x_t")[:, :K].copy(), inp.as_f32("x_prev")[:, :K].copy()


def _sub_max(xt, xp):
    """M_i of every sub-channel, fp32 subtraction then |.|, as [T x K]."""
    d = np.abs(xt.astype(np.float32) - xp.astype(np.float32))
    return d.reshape(-1, 16, d.shape[1]).max(axis=1)


def test_base_is_the_minimum_nonzero_sub_channel_max(orc):
    xt, xp = _small()
    # make some sub-channels exactly stationary: they must not enter the minimum
    xt[:16, :5] = xp[:16, :5]
    q = orc.quantize_dyn(xt, xp, -4)
    mx = _sub_max(xt, xp)
    assert (mx == 0).sum() >= 5
    assert q.base == float(mx[mx > 0].min())
    # the sub-channel holding the minimum gets PoT 0
    t, k = np.argwhere(mx == mx[mx > 0].min())[0]
    assert q.pot[t, k] == 0


@pytest.mark.parametrize("thr_lb,t0,force", [(-4, 0, 0), (-6, 1, 0), (-4, 0, 8), (-3, -1, 0)])
def test_pot_widths_and_codes_by_exact_arithmetic(orc, thr_lb, t0, force):
    xt, xp = _small(M=32, K=32)
    q = orc.quantize_dyn(xt, xp, thr_lb, t0, force)
    base = Fraction(q.base)
    dx = xt.astype(np.float32) - xp.astype(np.float32)
    mx = _sub_max(xt, xp)
    for t in range(mx.shape[0]):
        for k in range(mx.shape[1]):
            m = Fraction(float(mx[t, k]))
            P = 0
            while m > base * 2 ** P:
                P += 1
            assert q.pot[t, k] == P
            if force:
                b = force
            else:
                b = next((2 + 2 * n for n in range(3) if m <= Fraction(2) ** (thr_lb + t0 + 2 * n)), 8)
            assert q.bits[t, k] == b
            assert q.fpot[t, k] == b - 2 - P
            for i in range(16):
                u = np.float32(dx[16 * t + i, k]) / np.float32(q.base)  # IEEE fp32 division
                code = round(Fraction(float(u)) * Fraction(2) ** (b - 2 - P))  # ties to even
                assert q.codes[16 * t + i, k] == code
                assert abs(code) <= 2 ** (b - 2)
    assert (q.g_ref == q.fpot.max(axis=1)).all()


def test_power_of_two_minimum_reduces_to_the_static_quantizer(orc):
    """When the smallest M_i is exactly 2^L, the dynamic base equals the static
    base 2^L: the same widths, codes, accumulators and Y; the FPoT tags differ
    by the constant 2L (absolute against relative FPoT)."""
    rng = np.random.default_rng(5)
    M, K, N, L = 48, 64, 24, -6
    # X_{t-1} = 0, so dX = X_t exactly; every sub-channel max at least 2^(L+1),
    # one sub-channel exactly 2^L
    xp = np.zeros((M, K), np.float32)
    dx = (rng.uniform(1, 40, (M, K)) * np.sign(rng.standard_normal((M, K))) * 2.0 ** (L + 1)).astype(np.float32)
    dx[16:32, 7] = 0
    dx[20, 7] = -(2.0 ** L)
    xt = dx.copy()
    qd = orc.quantize_dyn(xt, xp, L)
    qs = orc.quantize(xt, xp, L)
    assert qd.base == 2.0 ** L
    assert np.array_equal(qd.codes, qs.codes) and np.array_equal(qd.bits, qs.bits)
    assert np.array_equal(qd.fpot.astype(int) - 2 * L, qs.fpot.astype(int))
    w = rng.integers(-127, 128, (N, K)).astype(np.int8)
    ws = rng.uniform(0.001, 0.01, N).astype(np.float32)
    yp = rng.standard_normal((M, N)).astype(np.float32)
    ad, as_ = orc.acc_direct(qd, w), orc.acc_direct(qs, w)
    assert np.array_equal(ad, as_)
    assert np.array_equal(orc.acc_slices(qd, w), ad)  # the encoded stream with relative tags
    for bf in (False, True):
        assert np.array_equal(orc.epilogue_dyn_f32(ad, qd.g_ref, qd.base, ws, yp, bf),
                              orc.epilogue_f32(as_, qs.g_ref, L, ws, yp, bf))


@pytest.mark.parametrize("kind", ["cfg2", "adversarial"])
def test_error_bound_tiny(orc, kind):
    """|dY - dX W_deq| <= sum_k (step/2 + |dX| 2^-24) |W_deq| with step = base 2^-FPoT."""
    if kind == "cfg2":
        xt, xp = _small(M=48, K=64)
        inp = synth.make_layer(2, 0, M=48)
        w, ws = inp.w_q[:40, :64], inp.w_scale[:40]
    else:
        inp = synth.adversarial_layer(48, 64, 40, seed=13, spread=20)
        xt, xp, w, ws = inp.as_f32("x_t"), inp.as_f32("x_prev"), inp.w_q, inp.w_scale
    q = orc.quantize_dyn(xt, xp, -4)
    acc = orc.acc_direct(q, np.ascontiguousarray(w))
    dy = acc.astype(np.float64) * np.repeat(np.exp2(-q.g_ref.astype(np.float64)), 16)[:, None] * q.base \
        * ws.astype(np.float64)[None, :]
    dx = (xt.astype(np.float32) - xp.astype(np.float32)).astype(np.float64)
    w_deq = w.astype(np.float64).T * ws.astype(np.float64)[None, :]
    exact = dx @ w_deq
    step = np.repeat(q.base * np.exp2(-q.fpot.astype(np.float64)), 16, axis=0)
    bound = (step / 2 + np.abs(dx) * 2.0 ** -24) @ np.abs(w_deq)
    assert (np.abs(dy - exact) <= bound * (1 + 1e-9) + 1e-12).all()
    assert np.abs(dy - exact).mean() < 0.5 * bound.mean()


def test_stationary_input(orc):
    xt, _ = _small()
    q = orc.quantize_dyn(xt, xt.copy(), -4)
    assert q.base == 1.0 and q.status == 0
    assert not q.codes.any() and (q.pot == 0).all()
    yp = np.random.default_rng(1).standard_normal((xt.shape[0], 16)).astype(np.float32)
    acc = np.zeros((xt.shape[0], 16), np.int64)
    assert np.array_equal(orc.epilogue_dyn_f32(acc, q.g_ref, q.base, np.ones(16, np.float32), yp, False), yp)


def test_nonfinite_sub_channel_is_excluded_and_flagged(orc):
    xt, xp = _small()
    xt[3, 2] = np.inf
    q = orc.quantize_dyn(xt, xp, -4)
    assert q.status & orc.ST_NONFINITE
    assert not q.codes[:16, 2].any()
    mx = _sub_max(xt, xp)
    mx[0, 2] = 0
    assert q.base == float(mx[mx > 0].min())
