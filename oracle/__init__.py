"""CPU oracle for the FMDQ differential linear layer -- TEST INFRASTRUCTURE.

Plain, slow and exact restatement of DSTAR's fine-grained mixed-precision
differential quantization (section 3.1, Eqs. 1-5; computation-flow steps 1-5
of Fig. 5) and of the MPU epilogue (section 4.2 inverse quantization and
accumulation units; section 4.3 reverse differential).  Only the tests, the
smoke check and the CPU-baseline leg of the benchmark may import this module.
It shares no code with the CUDA library and never calls it.

Every function takes and returns numpy arrays.  Floating-point inputs are fp32
arrays; bf16 data is widened exactly with :func:`bf16_to_f32` first.

Parity status of each function (what pins it, see tests/test_oracle_pins.py):
  quantize      -- worked PoT example (section 3.1, step 1), boundary cases,
                   rounding ties, closed form under forced 8/2 bits, slice
                   reassembly over every code, layout invariants.
  acc_slices    -- the value-70 example of section 3.1 step 2, equality with
                   acc_direct, the non-identity without shifts.
  acc_direct    -- equality with a numpy int64 matmul of the shifted codes.
  epilogue_f32  -- bounded against epilogue_f64 and against the dense fp64
                   product within the quantization error bound.
  quantize_dyn  -- (dynamic base) base equal to a brute-force minimum of the
                   nonzero M_i; PoT against exact rational comparisons; equal
                   to the static quantizer when the minimum is a power of two;
                   the error bound on tiny shapes.
  epilogue_dyn_f32 -- equal to epilogue_f32 when the base is a power of two.
  gelu          -- GELU(0) = 0, GELU(1) = Phi(1), GELU(y) - GELU(-y) = y,
                   against Python's math.erfc element by element, and
                   against math.erf away from the negative tail.
  ffn_gelu      -- composition of the pinned pieces above.
  quant_rows    -- brute force per element, the 127 bound, the error bound.
  masked_softmax -- rows sum to 1 over kept entries, pruned entries 0,
                   agreement with a numpy softmax of the kept entries, shift
                   invariance.
  sar_attention -- composition of the pinned pieces; its dense-mask output
                   within the quantization error of a plain fp64 attention.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

TILE = 16
ST_NONFINITE = 1
ST_RANGE = 2

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        ci = ctypes.c_int
        lib.fmdq_orc_quantize.argtypes = [P, P, i64, i64, ci, ci, ci] + [P] * 11
        lib.fmdq_orc_quantize.restype = ci
        lib.fmdq_orc_acc_slices.argtypes = [i64, i64, i64] + [P] * 10
        lib.fmdq_orc_acc_slices.restype = None
        lib.fmdq_orc_acc_direct.argtypes = [i64, i64, i64] + [P] * 6
        lib.fmdq_orc_acc_direct.restype = None
        lib.fmdq_orc_epilogue_f32.argtypes = [i64, i64, P, P, ci, P, P, ci, P, P]
        lib.fmdq_orc_epilogue_f32.restype = None
        lib.fmdq_orc_epilogue_f64.argtypes = [i64, i64, P, P, ci, P, P, P, P]
        lib.fmdq_orc_epilogue_f64.restype = None
        lib.fmdq_orc_bf16_to_f32.argtypes = [P, i64, P]
        lib.fmdq_orc_f32_to_bf16.argtypes = [P, i64, P]
        lib.fmdq_orc_slice_digit.argtypes = [ctypes.c_uint32, ci, ci]
        lib.fmdq_orc_slice_digit.restype = ci
        lib.fmdq_orc_pot_max.restype = ci
        lib.fmdq_orc_quantize_dyn.argtypes = [P, P, i64, i64, ci, ci, ci] + [P] * 12
        lib.fmdq_orc_quantize_dyn.restype = ci
        lib.fmdq_orc_epilogue_dyn_f32.argtypes = [i64, i64, P, P, ctypes.c_float, P, P, ci, P]
        lib.fmdq_orc_epilogue_dyn_f32.restype = None
        lib.fmdq_orc_gelu.argtypes = [P, i64, ci, P]
        lib.fmdq_orc_gelu.restype = None
        lib.fmdq_orc_quant_rows.argtypes = [P, i64, i64, P, P]
        lib.fmdq_orc_quant_rows.restype = None
        lib.fmdq_orc_masked_softmax.argtypes = [P, i64, i64, P, i64, i64, P]
        lib.fmdq_orc_masked_softmax.restype = None
        lib.fmdq_orc_set_threads.argtypes = [ci]
        lib.fmdq_orc_set_threads.restype = None
        lib.fmdq_orc_max_threads.restype = ci
        _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def pot_max() -> int:
    return _load().fmdq_orc_pot_max()


def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    _load().fmdq_orc_bf16_to_f32(_p(h), h.size, _p(out))
    return out


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, np.uint16)
    _load().fmdq_orc_f32_to_bf16(_p(f), f.size, _p(out))
    return out


def slice_digit(field: int, j: int, b: int) -> int:
    return _load().fmdq_orc_slice_digit(field, j, b)


class Quantized:
    """Everything steps 1-4 produce for one call."""

    def __init__(self, M, K):
        T = M // TILE
        cap = 4 * K
        self.M, self.K, self.T, self.cap = M, K, T, cap
        self.codes = np.zeros((M, K), np.int8)
        self.bits = np.zeros((T, K), np.int8)
        self.fpot = np.zeros((T, K), np.int8)
        self.pot = np.zeros((T, K), np.int16)
        self.g_ref = np.zeros(T, np.int32)
        self.count = np.zeros(T, np.int32)
        self.rec_word = np.zeros((T, cap), np.uint32)
        self.rec_k = np.zeros((T, cap), np.uint16)
        self.rec_tag = np.zeros((T, cap), np.int8)
        self.rec_j = np.zeros((T, cap), np.uint8)
        self.shift = np.zeros((T, cap), np.int8)
        self.status = 0


def quantize(x_t: np.ndarray, x_prev: np.ndarray, lb: int, t0: int = 0, force_bits: int = 0) -> Quantized:
    """Steps 1-4 of the computation flow for fp32 inputs [M x K], base = 2^lb."""
    x_t = np.ascontiguousarray(x_t, np.float32)
    x_prev = np.ascontiguousarray(x_prev, np.float32)
    M, K = x_t.shape
    assert x_prev.shape == (M, K) and M % TILE == 0
    q = Quantized(M, K)
    q.status = _load().fmdq_orc_quantize(
        _p(x_t), _p(x_prev), M, K, lb, t0, force_bits, _p(q.codes), _p(q.bits), _p(q.fpot), _p(q.pot),
        _p(q.g_ref), _p(q.count), _p(q.rec_word), _p(q.rec_k), _p(q.rec_tag), _p(q.rec_j), _p(q.shift))
    return q


def quantize_dyn(x_t: np.ndarray, x_prev: np.ndarray, thr_lb: int, t0: int = 0,
                 force_bits: int = 0) -> Quantized:
    """Steps 1-4 with the dynamic base (FMDQ-DYN): base = the minimum nonzero
    M_i of the call (first pass), widths from the predefined thresholds
    Thr_N = 2^(thr_lb + t0 + 2N); `fpot` holds FPoT relative to the base and
    `base` the base itself (fp32)."""
    x_t = np.ascontiguousarray(x_t, np.float32)
    x_prev = np.ascontiguousarray(x_prev, np.float32)
    M, K = x_t.shape
    assert x_prev.shape == (M, K) and M % TILE == 0
    q = Quantized(M, K)
    base = np.zeros(1, np.float32)
    q.status = _load().fmdq_orc_quantize_dyn(
        _p(x_t), _p(x_prev), M, K, thr_lb, t0, force_bits, _p(base), _p(q.codes), _p(q.bits), _p(q.fpot),
        _p(q.pot), _p(q.g_ref), _p(q.count), _p(q.rec_word), _p(q.rec_k), _p(q.rec_tag), _p(q.rec_j),
        _p(q.shift))
    q.base = float(base[0])
    return q


def epilogue_dyn_f32(acc: np.ndarray, g_ref: np.ndarray, base: float, w_scale: np.ndarray, y_prev: np.ndarray,
                     out_bf16: bool) -> np.ndarray:
    """Y_t = Y_{t-1} + acc * 2^-g_ref * base * w_scale in the fixed fp32 order (dynamic base)."""
    acc = np.ascontiguousarray(acc, np.int64)
    M, N = acc.shape
    w_scale = np.ascontiguousarray(w_scale, np.float32)
    y_prev = np.ascontiguousarray(y_prev, np.float32)
    g_ref = np.ascontiguousarray(g_ref, np.int32)
    out = np.zeros((M, N), np.float32)
    _load().fmdq_orc_epilogue_dyn_f32(M, N, _p(acc), _p(g_ref), float(np.float32(base)), _p(w_scale), _p(y_prev),
                                      int(out_bf16), _p(out))
    return out


def linear_dyn(x_t, x_prev, y_prev, w_q, w_scale, thr_lb, t0=0, force_bits=0, out_bf16=True):
    """The whole differential linear with the dynamic base: (Quantized, acc, y_out)."""
    q = quantize_dyn(x_t, x_prev, thr_lb, t0, force_bits)
    acc = acc_direct(q, w_q)
    y = epilogue_dyn_f32(acc, q.g_ref, q.base, w_scale, y_prev, out_bf16)
    return q, acc, y


def _mask(T, tiles):
    if tiles is None:
        return None
    m = np.zeros(T, np.uint8)
    m[np.asarray(tiles, dtype=np.int64)] = 1
    return m


def acc_slices(q: Quantized, w_q: np.ndarray, tiles=None) -> np.ndarray:
    """Step 5: shift-aligned accumulation over the encoded stream (int64 [M x N])."""
    w_q = np.ascontiguousarray(w_q, np.int8)
    N, K = w_q.shape
    assert K == q.K
    acc = np.zeros((q.M, N), np.int64)
    _load().fmdq_orc_acc_slices(q.M, q.K, N, _p(q.rec_word), _p(q.rec_k), _p(q.rec_tag), _p(q.rec_j),
                                _p(q.count), _p(q.bits), _p(q.g_ref), _p(w_q), _p(_mask(q.T, tiles)),
                                _p(acc))
    return acc


def acc_direct(q: Quantized, w_q: np.ndarray, tiles=None) -> np.ndarray:
    """The accumulator by its definition, sum_k code * 2^(g_ref - FPoT) * w (int64 [M x N])."""
    w_q = np.ascontiguousarray(w_q, np.int8)
    N, K = w_q.shape
    assert K == q.K
    acc = np.zeros((q.M, N), np.int64)
    _load().fmdq_orc_acc_direct(q.M, q.K, N, _p(q.codes), _p(q.fpot), _p(q.g_ref), _p(w_q),
                                _p(_mask(q.T, tiles)), _p(acc))
    return acc


def epilogue_f32(acc: np.ndarray, g_ref: np.ndarray, lb: int, w_scale: np.ndarray, y_prev: np.ndarray,
                 out_bf16: bool, tiles=None) -> np.ndarray:
    """Y_t = Y_{t-1} + dequant(acc) in the fixed fp32 order; fp32 array of the output values."""
    acc = np.ascontiguousarray(acc, np.int64)
    M, N = acc.shape
    w_scale = np.ascontiguousarray(w_scale, np.float32)
    y_prev = np.ascontiguousarray(y_prev, np.float32)
    g_ref = np.ascontiguousarray(g_ref, np.int32)
    out = np.zeros((M, N), np.float32)
    _load().fmdq_orc_epilogue_f32(M, N, _p(acc), _p(g_ref), lb, _p(w_scale), _p(y_prev), int(out_bf16),
                                  _p(_mask(M // TILE, tiles)), _p(out))
    return out


def epilogue_f64(acc: np.ndarray, g_ref: np.ndarray, lb: int, w_scale: np.ndarray, y_prev: np.ndarray,
                 tiles=None) -> np.ndarray:
    acc = np.ascontiguousarray(acc, np.int64)
    M, N = acc.shape
    w_scale = np.ascontiguousarray(w_scale, np.float32)
    y_prev = np.ascontiguousarray(y_prev, np.float32)
    g_ref = np.ascontiguousarray(g_ref, np.int32)
    out = np.zeros((M, N), np.float64)
    _load().fmdq_orc_epilogue_f64(M, N, _p(acc), _p(g_ref), lb, _p(w_scale), _p(y_prev),
                                  _p(_mask(M // TILE, tiles)), _p(out))
    return out


def linear(x_t, x_prev, y_prev, w_q, w_scale, lb, t0=0, force_bits=0, out_bf16=True, tiles=None,
           path="direct"):
    """The whole differential linear: returns (Quantized, acc, y_out)."""
    q = quantize(x_t, x_prev, lb, t0, force_bits)
    acc = acc_direct(q, w_q, tiles) if path == "direct" else acc_slices(q, w_q, tiles)
    y = epilogue_f32(acc, q.g_ref, lb, w_scale, y_prev, out_bf16, tiles)
    return q, acc, y


def gelu(y: np.ndarray, out_bf16: bool) -> np.ndarray:
    """GELU(y) = y * Phi(y) = 0.5 y erfc(-y / sqrt 2) in fp64, rounded to fp32 (then bf16 when out_bf16)."""
    y = np.ascontiguousarray(y, np.float32)
    out = np.empty_like(y)
    _load().fmdq_orc_gelu(_p(y), y.size, int(out_bf16), _p(out))
    return out


def ffn_gelu(x_t, x_prev, y1_prev, w1, w1_scale, h_prev, y2_prev, w2, w2_scale, lb, t0=0, force_bits=0,
             out_bf16=True):
    """The chained FFN pair with the GELU between the layers (section 4.3):
    layer 1 on (X_t, X_{t-1}), H_t = GELU(Y1_t), layer 2 on (H_t, H_{t-1}).
    Returns (q1, acc1, y1, h, q2, acc2, y2)."""
    q1, acc1, y1 = linear(x_t, x_prev, y1_prev, w1, w1_scale, lb, t0, force_bits, out_bf16)
    h = gelu(y1, out_bf16)
    q2, acc2, y2 = linear(h, h_prev, y2_prev, w2, w2_scale, lb, t0, force_bits, out_bf16)
    return q1, acc1, y1, h, q2, acc2, y2


def quant_rows(x: np.ndarray):
    """Symmetric per-row int8: scale = max|row|/127, q = rne(x/scale); returns (q int8, scale fp32)."""
    x = np.ascontiguousarray(x, np.float32)
    rows, cols = x.shape
    q = np.zeros((rows, cols), np.int8)
    sc = np.zeros(rows, np.float32)
    _load().fmdq_orc_quant_rows(_p(x), rows, cols, _p(q), _p(sc))
    return q, sc


def masked_softmax(s: np.ndarray, mask: np.ndarray, blk: int) -> np.ndarray:
    """Row softmax over the kept blocks of a block mask (fp64, rounded to fp32); pruned entries 0."""
    s = np.ascontiguousarray(s, np.float32)
    rows, cols = s.shape
    mask = np.ascontiguousarray(mask, np.uint8)
    assert mask.shape == ((rows + blk - 1) // blk, (cols + blk - 1) // blk)
    out = np.zeros((rows, cols), np.float32)
    _load().fmdq_orc_masked_softmax(_p(s), rows, cols, _p(mask), blk, mask.shape[1], _p(out))
    return out


def sar_attention(q, k, v, mask, blk, lb_q, lb_p, scores_scale, p_cached=None):
    """Attention of one head with INT8 FMDQ operands and sparse attention reuse
    (sections 3.2 and 4.3).  q, k: [S x d]; v: [S x d]; mask [S/blk x S/blk].

    Cached step (p_cached None):
      K -> int8 per key (quant_rows); Q -> FMDQ with every width 8 and X_{t-1} = 0;
      scores = dequant(acc(Q codes, K codes)) with w_scale = fl32(k_scale * scores_scale);
      P = masked_softmax(scores); P -> FMDQ with every width 8 (the cached object).
    Reused step: the cached quantized P.
    Both: V^T -> int8 per head dimension; O = dequant(acc(P codes, V^T codes)).
    Returns dict(qQ, kq, ks, acc_s, scores, p, qP, vq, vs, acc_o, out)."""
    S, d = q.shape
    res = {}
    if p_cached is None:
        kq, ks = quant_rows(k)
        zeros_q = np.zeros_like(q, dtype=np.float32)
        qQ = quantize(q, zeros_q, lb_q, 0, 8)
        acc_s = acc_direct(qQ, kq)
        w_s = (ks * np.float32(scores_scale)).astype(np.float32)
        scores = epilogue_f32(acc_s, qQ.g_ref, lb_q, w_s, np.zeros((S, S), np.float32), False)
        p = masked_softmax(scores, mask, blk)
        qP = quantize(p, np.zeros_like(p), lb_p, 0, 8)
        res.update(qQ=qQ, kq=kq, ks=ks, acc_s=acc_s, scores=scores, p=p, qP=qP)
    else:
        qP = p_cached
        res.update(qP=qP)
    vq, vs = quant_rows(np.ascontiguousarray(v.T))
    acc_o = acc_direct(qP, vq)
    out = epilogue_f32(acc_o, qP.g_ref, lb_p, vs, np.zeros((S, vq.shape[0]), np.float32), False)
    res.update(vq=vq, vs=vs, acc_o=acc_o, out=out)
    return res


def n_threads() -> int:
    """Threads the oracle's loops use now."""
    return int(_load().fmdq_orc_max_threads())


def set_threads(n: int) -> None:
    """Run the oracle's loops on n threads (timing only; results do not change)."""
    _load().fmdq_orc_set_threads(int(n))
