"""Pins of the CPU oracle against what the paper and the mathematics fix.

The oracle (oracle/) is the parity reference of the CUDA path, so it is pinned
here to facts that do not come from itself: the paper's worked examples
(tests/golden/), closed forms, brute force over small domains, invariants,
numpy library routines and the quantization error bound.
"""
import math
import os

import numpy as np
import pytest

from differential_quantized_gemm_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kv(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split("=", 1)
        out[k] = v
    return out


def _tile_with_column(col_values, K=1, col=0, other=0.0):
    """A single 16-token tile whose channel `col` holds col_values (dx), x_prev = 0."""
    x_t = np.full((16, K), other, np.float32)
    x_t[:, col] = np.asarray(col_values, np.float32)
    return x_t, np.zeros_like(x_t)


def _pot_brute(mx, lb):
    """Smallest p >= 0 with mx <= 2^lb * 2^p (Eq. 3 with the static-base clamp)."""
    p = 0
    while mx > math.ldexp(1.0, lb + p):
        p += 1
    return p


# --------------------------------------------------------------- step 1 pins

def test_worked_example_pot(orc):
    g = _kv("worked_example_pot.txt")
    lb, t0 = int(g["base_log2"]), int(g["t0"])
    vals = np.linspace(-0.3, 0.5, 16).astype(np.float32)
    vals[3] = float(g["max_abs"])
    x_t, x_p = _tile_with_column(vals)
    q = orc.quantize(x_t, x_p, lb, t0)
    assert q.bits[0, 0] == int(g["bits"])
    assert 2 ** (q.bits[0, 0] - 2) == int(g["pceil"])
    assert q.pot[0, 0] == int(g["pot"])
    assert q.fpot[0, 0] == int(g["fpot"])
    assert math.ldexp(1.0, lb + int(q.fpot[0, 0])) == float(g["scale"])  # Eq. 5
    assert q.codes[3, 0] == int(g["code_of_max"])
    # with s_i = 1 every code is the value rounded half-to-even
    assert np.array_equal(q.codes[:, 0], np.rint(vals).astype(np.int8))


@pytest.mark.parametrize("lb", [-10, -4, 0, 3])
@pytest.mark.parametrize("P", [0, 1, 3, 6, 9])
def test_pot_boundaries(orc, lb, P):
    base_pow = math.ldexp(1.0, lb + P)
    # exactly at base * 2^P -> PoT = P (ceil of an exact integer)
    q = orc.quantize(*_tile_with_column([base_pow] + [0.0] * 15), lb)
    assert q.pot[0, 0] == P
    # one ulp above -> PoT = P + 1
    above = np.nextafter(np.float32(base_pow), np.float32(np.inf))
    q = orc.quantize(*_tile_with_column([above] + [0.0] * 15), lb)
    assert q.pot[0, 0] == P + 1
    assert q.pot[0, 0] == _pot_brute(float(above), lb)


def test_pot_below_base_and_zero(orc):
    lb = -4
    q = orc.quantize(*_tile_with_column([0.0625, -0.03] + [0.0] * 14), lb)
    assert q.pot[0, 0] == 0 and q.bits[0, 0] == 2
    q = orc.quantize(*_tile_with_column([0.0] * 16), lb)
    assert q.pot[0, 0] == 0 and not q.codes.any()


def test_rounding_ties_to_even(orc):
    # forced 8 bits, base 1, max 64 -> PoT 6, FPoT 0, s_i = 1: codes = rne(dx)
    col = [0.5, 1.5, -2.5, 2.5, -0.5, 3.5, 64.0] + [0.0] * 9
    q = orc.quantize(*_tile_with_column(col), 0, force_bits=8)
    assert q.pot[0, 0] == 6 and q.fpot[0, 0] == 0
    assert list(q.codes[:7, 0]) == [0, 2, -2, 2, 0, 4, 64]


@pytest.mark.parametrize("t0", [0, 2, 5])
def test_threshold_binning(orc, t0):
    """Thr_N = Thr_0 * 2^(2N): bins of PoT at t0, t0+2, t0+4 (section 3.1)."""
    lb = -4
    for P in range(0, t0 + 9):
        mx = math.ldexp(1.0, lb + P)
        q = orc.quantize(*_tile_with_column([mx] + [0.0] * 15), lb, t0)
        expect = 2 if P <= t0 else 4 if P <= t0 + 2 else 6 if P <= t0 + 4 else 8
        assert q.bits[0, 0] == expect, (P, t0)
        # Eq. 4 with PCeil = 2^(b-2)
        assert q.fpot[0, 0] == (expect - 2) - 2 * lb - P


def test_forced_8bit_closed_form(orc):
    """Invariant I3: with every sub-channel at 8 bits the codes are plain per
    sub-channel power-of-two quantization rne(dx / (base * 2^(PoT - 6)))."""
    rng = np.random.default_rng(5)
    M, K, lb = 64, 24, -4
    mags = np.exp2(rng.uniform(-6, 6, size=(M // 16, K)))
    dx = (rng.standard_normal((M, K)) * np.repeat(mags, 16, axis=0)).astype(np.float32)
    q = orc.quantize(dx, np.zeros_like(dx), lb, force_bits=8)
    for t in range(M // 16):
        for k in range(K):
            col = dx[16 * t:16 * t + 16, k].astype(np.float64)
            P = _pot_brute(np.abs(col).max(), lb)
            step = math.ldexp(1.0, lb + P - 6)
            assert np.array_equal(q.codes[16 * t:16 * t + 16, k], np.rint(col / step).astype(np.int8))
    assert (q.bits == 8).all()


def test_forced_2bit_codes_ternary(orc):
    rng = np.random.default_rng(6)
    dx = rng.standard_normal((32, 40)).astype(np.float32)
    q = orc.quantize(dx, np.zeros_like(dx), -4, force_bits=2)
    assert set(np.unique(q.codes)) <= {-1, 0, 1}
    assert (q.count == 40).all()


def test_no_clipping_needed(orc):
    """Invariant I0: |code| <= PCeil = 2^(b-2) for every element."""
    inp = synth.adversarial_layer(64, 64, 16, seed=3)
    q = orc.quantize(inp.as_f32("x_t"), inp.as_f32("x_prev"), -4)
    lim = np.repeat(2 ** (q.bits.astype(np.int32) - 2), 16, axis=0)
    assert (np.abs(q.codes.astype(np.int32)) <= lim).all()
    assert q.status == 0


def test_nonfinite_and_range_status(orc):
    x_t, x_p = _tile_with_column([np.inf] + [0.0] * 15, K=2)
    q = orc.quantize(x_t, x_p, -4)
    assert q.status & orc.ST_NONFINITE and not q.codes.any()
    big = math.ldexp(1.0, -4 + orc.pot_max() + 1)
    q = orc.quantize(*_tile_with_column([big] + [0.0] * 15), -4)
    assert q.status & orc.ST_RANGE


# --------------------------------------------------------------- step 2 pins

@pytest.mark.parametrize("b", [2, 4, 6, 8])
def test_slices_reassemble_every_code(orc, b):
    """Invariant I1: the 2-bit slices of every code reassemble it exactly,
    sum_j d_j 4^j = q (section 3.1 step 2 identity)."""
    lim = 2 ** (b - 2)
    for qv in range(-lim, lim + 1):
        u = qv & ((1 << b) - 1)
        digits = [orc.slice_digit((u >> (2 * j)) & 3, j, b) for j in range(b // 2)]
        assert sum(d * 4 ** j for j, d in enumerate(digits)) == qv
        assert all(0 <= d <= 3 for d in digits[:-1]) and -2 <= digits[-1] <= 1


@pytest.mark.parametrize("b", [2, 4, 6, 8])
def test_slices_from_quantizer_reassemble(orc, b):
    """The encoded stream of a tile whose codes cover the whole range of b bits
    reassembles to exactly those codes (codes chosen with s_i = 1)."""
    lim = 2 ** (b - 2)
    vals = list(range(-lim, lim + 1))
    ncol = (len(vals) + 14) // 15
    x_t = np.zeros((16, ncol), np.float32)
    for c in range(ncol):
        chunk = vals[15 * c:15 * c + 15]
        x_t[:len(chunk), c] = chunk
        x_t[15, c] = lim  # pins PoT = b - 2 so that s_i = 1
    q = orc.quantize(x_t, np.zeros_like(x_t), 0, force_bits=b)
    assert (q.fpot == 0).all()
    rebuilt = np.zeros((16, ncol), np.int64)
    for r in range(q.count[0]):
        k, j, w = int(q.rec_k[0, r]), int(q.rec_j[0, r]), int(q.rec_word[0, r])
        assert q.rec_tag[0, r] == q.fpot[0, k] - 2 * j
        for i in range(16):
            rebuilt[i, k] += orc.slice_digit((w >> (2 * i)) & 3, j, b) * 4 ** j
    assert np.array_equal(rebuilt, q.codes.astype(np.int64))


def _manual_tile(orc, records, K, N, bits_of_k):
    """Build a Quantized holding one tile with the given (tag, k, j, word) records."""
    q = orc.Quantized(16, K)
    for r, (tag, k, j, word) in enumerate(records):
        q.rec_tag[0, r], q.rec_k[0, r], q.rec_j[0, r], q.rec_word[0, r] = tag, k, j, word
    q.count[0] = len(records)
    for k, b in bits_of_k.items():
        q.bits[0, k] = b
    q.g_ref[0] = max(t for t, *_ in records)
    return q


def test_value_70_example(orc):
    """Section 3.1 step 2: 70 -> slices 1,0,1,2 with FPoT 1,3,5,7; ascending-FPoT
    accumulation with shifts gives 70 w."""
    g = _kv("slice_example_70.txt")
    value, b = int(g["value"]), int(g["bits"])
    slices = [int(s) for s in g["slices_high_to_low"].split(",")]
    fpots = [int(s) for s in g["fpot_high_to_low"].split(",")]
    u = value & ((1 << b) - 1)
    assert [(u >> (2 * j)) & 3 for j in (3, 2, 1, 0)] == slices
    assert [fpots[-1] - 2 * j for j in (3, 2, 1, 0)] == fpots
    w = np.array([[37], [-101]], np.int8).reshape(2, 1)
    records = [(fpots[i], 0, 3 - i, slices[i]) for i in range(4)]  # token 0 carries the value
    q = _manual_tile(orc, records, K=1, N=2, bits_of_k={0: b})
    acc = orc.acc_slices(q, w)
    assert list(acc[0]) == [value * 37, value * -101]
    assert not acc[1:].any()
    # the non-identity of step 2: without the shifts the products do not add up
    flat = [(fpots[-1], 0, 3 - i, slices[i]) for i in range(4)]
    q2 = _manual_tile(orc, flat, K=1, N=2, bits_of_k={0: b})
    assert orc.acc_slices(q2, w)[0, 0] == sum(slices) * 37 != value * 37


def test_fig11_shift_counts(orc):
    """Encoding (step 4): shifts are adjacent FPoT differences; the Fig. 11 block
    changes FPoT between ID 5 and 6."""
    g = _kv("fig11_meta.txt")
    fp = [int(s) for s in g["fpot"].split(",")]
    want = [int(s) for s in g["shifts"].split(",")]
    # a tile with 6 channels at FPoT 4 and 2 at FPoT 5 (all 2-bit: one slice each)
    lb = 0
    # 2-bit with FPoT = -2*lb - PoT -> PoT = -FPoT; use lb = -4: FPoT = 8 - PoT
    lb = -4
    pots = [8 - f for f in fp]
    x_t = np.zeros((16, len(fp)), np.float32)
    for k, P in enumerate(pots):
        x_t[0, k] = math.ldexp(1.0, lb + P)
    q = orc.quantize(x_t, np.zeros_like(x_t), lb, t0=10)
    assert list(q.rec_tag[0, :q.count[0]]) == sorted(fp)
    assert list(q.shift[0, :q.count[0]]) == want


# ------------------------------------------------------- step 3-5 invariants

def _layout_invariants(q):
    for t in range(q.T):
        n = q.count[t]
        assert n == int(q.bits[t].astype(np.int32).sum() // 2)
        tags = q.rec_tag[t, :n].astype(np.int32)
        ks = q.rec_k[t, :n].astype(np.int32)
        assert (np.diff(tags) >= 0).all()
        same = np.diff(tags) == 0
        assert (np.diff(ks)[same] > 0).all()
        assert (q.shift[t, :n] >= 0).all() and q.shift[t, 0] == 0
        assert np.array_equal(q.shift[t, 1:n], np.diff(tags))
        seen = set(zip(ks.tolist(), q.rec_j[t, :n].tolist()))
        assert len(seen) == n
        want = {(k, j) for k in range(q.K) for j in range(int(q.bits[t, k]) // 2)}
        assert seen == want
        assert q.g_ref[t] == q.fpot[t].max() == tags.max()


@pytest.mark.parametrize("kind", ["random", "adversarial", "force8", "force2"])
def test_layout_and_shift_aligned_equals_direct(orc, kind):
    """Invariants I2 and I5: the slice-stream accumulation (ascending FPoT with
    shifts) equals the direct shifted-code accumulation bit for bit, and the
    grouped layout is a sorted permutation of all slices."""
    if kind == "random":
        inp = synth.make_layer(3, layer=1, M=64)
        inp = synth.LayerInputs(synth.LayerSpec("s", 64, 48, 24, "bf16", -4), inp.x_t[:, :48],
                                inp.x_prev[:, :48], inp.y_prev[:, :24], inp.w_q[:24, :48], inp.w_scale[:24])
        fb = 0
    else:
        inp = synth.adversarial_layer(64, 48, 24, seed=11, spread=30)
        fb = {"adversarial": 0, "force8": 8, "force2": 2}[kind]
    q = orc.quantize(inp.as_f32("x_t"), inp.as_f32("x_prev"), -4, force_bits=fb)
    _layout_invariants(q)
    a1 = orc.acc_slices(q, inp.w_q)
    a2 = orc.acc_direct(q, inp.w_q)
    assert np.array_equal(a1, a2)
    if kind == "adversarial":
        assert len(np.unique(q.fpot)) >= 8  # many FPoT groups per tile


def test_direct_equals_numpy_matmul(orc):
    inp = synth.adversarial_layer(48, 40, 20, seed=12, spread=16)
    q = orc.quantize(inp.as_f32("x_t"), inp.as_f32("x_prev"), -4)
    shift = np.repeat(q.g_ref[:, None] - q.fpot.astype(np.int64), 16, axis=0)
    v = q.codes.astype(np.int64) << shift
    assert np.array_equal(orc.acc_direct(q, inp.w_q), v @ inp.w_q.astype(np.int64).T)


# ------------------------------------------------------------ epilogue pins

@pytest.mark.parametrize("kind", ["cfg1", "cfg2", "adversarial"])
def test_error_bound_tiny(orc, kind):
    """Invariant I4: on tiny shapes the quantized dY differs from the exact
    dX W_deq by at most the sum of half-steps times |W_deq| (plus fp rounding)."""
    if kind == "cfg1":
        inp = synth.make_layer(1, M=32)
        inp.w_q, inp.w_scale = inp.w_q[:32, :64], inp.w_scale[:32]
        inp.x_t, inp.x_prev = inp.x_t[:, :64], inp.x_prev[:, :64]
        lb = -10
    elif kind == "cfg2":
        inp = synth.make_layer(2, M=48)
        inp.w_q, inp.w_scale = inp.w_q[:40, :64], inp.w_scale[:40]
        inp.x_t, inp.x_prev = inp.x_t[:, :64], inp.x_prev[:, :64]
        lb = -4
    else:
        inp = synth.adversarial_layer(48, 64, 40, seed=13, spread=20)
        lb = -4
    xt, xp = inp.as_f32("x_t"), inp.as_f32("x_prev")
    q = orc.quantize(xt, xp, lb)
    acc = orc.acc_direct(q, inp.w_q)
    N = inp.w_q.shape[0]
    zeros = np.zeros((xt.shape[0], N), np.float32)
    dy = orc.epilogue_f64(acc, q.g_ref, lb, inp.w_scale, zeros)
    dx = xt.astype(np.float32) - xp.astype(np.float32)
    w_deq = inp.w_q.astype(np.float64).T * inp.w_scale.astype(np.float64)[None, :]
    exact = dx.astype(np.float64) @ w_deq
    step = np.repeat(np.exp2(-lb - q.fpot.astype(np.float64)), 16, axis=0)
    bound = (step / 2) @ np.abs(w_deq)
    slop = 1e-12 * (np.abs(dx.astype(np.float64)) @ np.abs(w_deq) + 1)
    assert (np.abs(dy - exact) <= bound + slop).all()
    # and the bound is not vacuous: the error is mostly well inside it
    assert np.abs(dy - exact).mean() < 0.5 * bound.mean()


@pytest.mark.parametrize("out_bf16", [False, True])
def test_epilogue_fp32_order_within_fp64(orc, out_bf16):
    inp = synth.make_layer(2, M=64)
    K = 128
    N = 64
    xt, xp = inp.as_f32("x_t")[:, :K], inp.as_f32("x_prev")[:, :K]
    w_q, w_s = inp.w_q[:N, :K], inp.w_scale[:N]
    y_prev = inp.as_f32("y_prev")[:, :N]
    q = orc.quantize(xt, xp, -4)
    acc = orc.acc_direct(q, w_q)
    y32 = orc.epilogue_f32(acc, q.g_ref, -4, w_s, y_prev, out_bf16).astype(np.float64)
    y64 = orc.epilogue_f64(acc, q.g_ref, -4, w_s, y_prev)
    dy = y64 - y_prev.astype(np.float64)
    tol = 3 * 2.0 ** -24 * (np.abs(dy) + np.abs(y64)) + 1e-30
    if out_bf16:
        tol = tol + 2.0 ** -8 * np.abs(y64)
    assert (np.abs(y32 - y64) <= tol).all()
    if out_bf16:
        # the result is a bf16 value
        assert np.array_equal(orc.bf16_to_f32(orc.f32_to_bf16(y32.astype(np.float32))), y32.astype(np.float32))


def test_stationary_input_keeps_output(orc):
    """Invariant I6: dX = 0 -> zero codes, zero accumulator, Y_t == Y_{t-1} bit for bit."""
    inp = synth.make_layer(2, M=32)
    xp = inp.as_f32("x_prev")[:, :96]
    q = orc.quantize(xp, xp, -4)
    assert not q.codes.any()
    acc = orc.acc_direct(q, inp.w_q[:50, :96])
    assert not acc.any()
    y_prev = inp.as_f32("y_prev")[:, :50]
    y = orc.epilogue_f32(acc, q.g_ref, -4, inp.w_scale[:50], y_prev, True)
    assert np.array_equal(y, y_prev)


def test_bf16_helpers_against_numpy(orc):
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(4096) * np.exp2(rng.uniform(-20, 20, 4096))).astype(np.float32)
    h = orc.f32_to_bf16(x)
    assert np.array_equal(h, synth.to_bf16_bits(x))
    back = orc.bf16_to_f32(h)
    # nearest bf16: error at most half a bf16 ulp
    assert (np.abs(back - x) <= np.abs(x) * 2.0 ** -8).all()
