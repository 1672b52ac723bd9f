"""ctypes binding of libdstar_fmdq.so (the C ABI in include/dstar_fmdq.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  torch tensors supply device memory and the current stream.  If the
library has not been built, every entry point raises instead of computing
anything another way.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "_lib", "libdstar_fmdq.so")

DSTAR_OK = 0
ERR = {-1: "INVALID_ARG", -2: "WORKSPACE", -3: "CUDA", -4: "UNSUPPORTED"}
STATUS_NONFINITE, STATUS_RANGE, STATUS_TIMEOUT = 1, 2, 4
F32, BF16, I8 = 0, 1, 2
FLAG_NO_XPREV_REFRESH = 1
FLAG_SLICE_PATH = 2
FLAG_DYNAMIC_BASE = 4
# slice-GEMM tile forms (a tuning override in flags bits 8..10; 0 = the library's choice)
TILE_128x128, TILE_128x256, TILE_PAIR_256x256, TILE_PAIR_256x128 = 1, 2, 3, 4
TILE_SHIFT = 8


def tile_flag(form: int) -> int:
    """The flags bits that make a call use slice-GEMM tile form `form`."""
    return int(form) << TILE_SHIFT


TILE = 16
POT_MAX = 32
K_MAX = 8192

EXPORTED = [
    "dstar_fmdq_version", "dstar_fmdq_error_string", "dstar_fmdq_last_error", "dstar_fmdq_workspace_size",
    "dstar_fmdq_workspace_layout", "dstar_fmdq_workspace_init", "dstar_fmdq_linear", "dstar_fmdq_quantize",
    "dstar_fmdq_slice_gemm", "dstar_fmdq_status", "dstar_fmdq_selftest_wait", "dstar_fmdq_linear_noalloc",
    "dstar_fmdq_ffn_gelu", "dstar_sar_workspace_size", "dstar_sar_workspace_layout", "dstar_sar_workspace_init",
    "dstar_sar_attention", "dstar_sar_status", "dstar_fmdq_gemm_tile", "dstar_fmdq_selftest_div",
]
SAR_BLOCK = 128
NOALLOC_SCRATCH_BYTES = 64 << 20


class DstarMat(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("ld", ctypes.c_int64)]


class TileCfg(ctypes.Structure):
    _fields_ = [("tile_tokens", ctypes.c_int32), ("thr0_log2", ctypes.c_int32), ("force_bits", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("debug_codes", ctypes.c_void_p), ("debug_acc", ctypes.c_void_p)]


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("total", "status", "plane0", "plane1", "fpot", "bits", "g_ref",
                                               "planes", "count", "mask1", "records")] + \
               [("mask_words", ctypes.c_int64), ("record_cap", ctypes.c_int64), ("dyn_base", ctypes.c_size_t)]


class SarCfg(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int64), ("seq", ctypes.c_int64), ("head_dim", ctypes.c_int64),
                ("block_mask", ctypes.c_void_p), ("scores_scale", ctypes.c_float), ("base_q", ctypes.c_float),
                ("base_p", ctypes.c_float), ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)]


class SarLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("total", "ws_p", "ws_q", "kq", "ks", "vqt", "vs", "scores", "probs")]


class DstarError(RuntimeError):
    pass


_lib = None


def lib():
    """The loaded CUDA library; raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DstarError(f"CUDA library not built ({LIB_PATH} missing); run "
                             "`python -m differential_quantized_gemm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64 = ctypes.c_void_p, ctypes.c_int64
        MP = ctypes.POINTER(DstarMat)
        L.dstar_fmdq_version.restype = ctypes.c_int
        L.dstar_fmdq_error_string.argtypes = [ctypes.c_int]
        L.dstar_fmdq_error_string.restype = ctypes.c_char_p
        L.dstar_fmdq_last_error.restype = ctypes.c_char_p
        L.dstar_fmdq_workspace_size.argtypes = [I64, I64, ctypes.POINTER(ctypes.c_size_t)]
        L.dstar_fmdq_workspace_layout.argtypes = [I64, I64, ctypes.POINTER(WsLayout)]
        L.dstar_fmdq_workspace_init.argtypes = [P, ctypes.c_size_t, P]
        L.dstar_fmdq_linear.argtypes = [MP, MP, MP, MP, P, ctypes.c_float, ctypes.POINTER(TileCfg), MP, P]
        L.dstar_fmdq_quantize.argtypes = [MP, MP, ctypes.c_float, ctypes.POINTER(TileCfg), P]
        L.dstar_fmdq_slice_gemm.argtypes = [MP, P, MP, ctypes.c_float, ctypes.POINTER(TileCfg), MP, P]
        L.dstar_fmdq_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
        L.dstar_fmdq_selftest_wait.argtypes = [P, ctypes.c_uint32, P]
        L.dstar_fmdq_linear_noalloc.argtypes = [MP, MP, MP, MP, P, ctypes.c_float, ctypes.POINTER(TileCfg), MP, P,
                                                P]
        L.dstar_fmdq_ffn_gelu.argtypes = [MP, MP, MP, MP, P, MP, MP, MP, MP, P, ctypes.c_float,
                                          ctypes.POINTER(TileCfg), ctypes.POINTER(TileCfg), P]
        L.dstar_sar_workspace_size.argtypes = [I64, I64, I64, ctypes.POINTER(ctypes.c_size_t)]
        L.dstar_sar_workspace_layout.argtypes = [I64, I64, I64, ctypes.POINTER(SarLayout)]
        L.dstar_sar_workspace_init.argtypes = [ctypes.POINTER(SarCfg), P]
        L.dstar_sar_attention.argtypes = [MP, MP, MP, ctypes.POINTER(SarCfg), ctypes.c_int, MP, P]
        L.dstar_sar_status.argtypes = [ctypes.POINTER(SarCfg), P, ctypes.POINTER(ctypes.c_uint32)]
        L.dstar_fmdq_selftest_div.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
        L.dstar_fmdq_gemm_tile.argtypes = [I64, I64, I64, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                           ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        for name in EXPORTED[3:]:
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int):
    if rc != DSTAR_OK:
        msg = lib().dstar_fmdq_last_error().decode()
        raise DstarError(f"{ERR.get(rc, rc)}: {msg}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.int8:
        return I8
    raise DstarError(f"unsupported dtype {t.dtype}")


def mat(t: torch.Tensor | None) -> DstarMat | None:
    """Describe a 2-D row-major tensor (unit column stride) for the C ABI."""
    if t is None:
        return None
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise DstarError("matrices must be 2-D with unit column stride")
    return DstarMat(t.data_ptr() if t.numel() else None, _dtype_code(t), 0, t.shape[0], t.shape[1],
                    t.stride(0) if t.shape[0] > 1 else max(t.shape[1], 1))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def workspace_size(M: int, K: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().dstar_fmdq_workspace_size(M, K, ctypes.byref(n)))
    return n.value


def workspace_layout(M: int, K: int) -> WsLayout:
    L = WsLayout()
    _check(lib().dstar_fmdq_workspace_layout(M, K, ctypes.byref(L)))
    return L


class Workspace:
    """Caller-owned device scratch for calls with up to M tokens and K channels."""

    def __init__(self, M: int, K: int, device="cuda", stream=None):
        self.M, self.K = M, K
        self.nbytes = workspace_size(M, K)
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-self.buf.data_ptr()) % 256
        self.buf = self.buf[off:off + self.nbytes]
        _check(lib().dstar_fmdq_workspace_init(ctypes.c_void_p(self.buf.data_ptr()), self.nbytes, _stream(stream)))

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def sections(self, M: int | None = None, K: int | None = None) -> dict:
        """Views of the quantizer outputs held in the workspace (for inspection)."""
        M = self.M if M is None else M
        K = self.K if K is None else K
        T = M // TILE
        L = workspace_layout(M, K)

        def view(off, n, dtype):
            nb = n * torch.tensor([], dtype=dtype).element_size()
            return self.buf[off:off + nb].view(dtype)

        return {
            "status": view(L.status, 1, torch.int32),
            "plane0": view(L.plane0, M * K, torch.int8).view(M, K),
            "plane1": view(L.plane1, M * K, torch.int8).view(M, K),
            "fpot": view(L.fpot, T * K, torch.int8).view(T, K),
            "bits": view(L.bits, T * K, torch.int8).view(T, K),
            "g_ref": view(L.g_ref, T, torch.int32),
            "planes": view(L.planes, T, torch.int32),
            "count": view(L.count, T, torch.int32),
            "mask1": view(L.mask1, T * L.mask_words, torch.int32).view(T, L.mask_words),
            "records": view(L.records, T * L.record_cap * 2, torch.int32).view(T, L.record_cap, 2),
            "dyn_base": view(L.dyn_base, 1, torch.float32),
        }


def _cfg(ws: Workspace, t0: int, force_bits: int, flags: int, debug_codes, debug_acc) -> TileCfg:
    return TileCfg(TILE, t0, force_bits, flags, ctypes.c_void_p(ws.ptr), ws.nbytes,
                   ctypes.c_void_p(debug_codes.data_ptr()) if debug_codes is not None else None,
                   ctypes.c_void_p(debug_acc.data_ptr()) if debug_acc is not None else None)


def linear(x_t, x_prev, y_prev, w_q, w_scale, base_scale: float, ws: Workspace, *, t0: int = 0,
           force_bits: int = 0, flags: int = 0, y_out=None, debug_codes=None, debug_acc=None, stream=None):
    """dstar_fmdq_linear: Y_t = Y_{t-1} + dequant(FMDQ(X_t - X_{t-1}) W); returns y_out (y_prev if None)."""
    if y_out is None:
        y_out = y_prev
    cfg = _cfg(ws, t0, force_bits, flags, debug_codes, debug_acc)
    mx, mp, my, mw, mo = mat(x_t), mat(x_prev), mat(y_prev), mat(w_q), mat(y_out)
    _check(lib().dstar_fmdq_linear(ctypes.byref(mx), ctypes.byref(mp), ctypes.byref(my), ctypes.byref(mw),
                                   ctypes.c_void_p(w_scale.data_ptr()), base_scale, ctypes.byref(cfg),
                                   ctypes.byref(mo), _stream(stream)))
    return y_out


def linear_noalloc(x_t, x_prev, y_prev, w_q, w_scale, base_scale: float, *, t0: int = 0, force_bits: int = 0,
                   flags: int = 0, y_out=None, status_out=None, debug_codes=None, debug_acc=None, stream=None):
    """dstar_fmdq_linear_noalloc: dstar_fmdq_linear with the library's static
    device scratch in place of a workspace, for callers that cannot allocate.
    status_out: optional int32/uint32 device tensor of one element that receives
    this call's status bits.  Returns y_out (y_prev if None)."""
    if y_out is None:
        y_out = y_prev
    cfg = TileCfg(TILE, t0, force_bits, flags, None, 0,
                  ctypes.c_void_p(debug_codes.data_ptr()) if debug_codes is not None else None,
                  ctypes.c_void_p(debug_acc.data_ptr()) if debug_acc is not None else None)
    mx, mp, my, mw, mo = mat(x_t), mat(x_prev), mat(y_prev), mat(w_q), mat(y_out)
    st = ctypes.c_void_p(status_out.data_ptr()) if status_out is not None else None
    _check(lib().dstar_fmdq_linear_noalloc(ctypes.byref(mx), ctypes.byref(mp), ctypes.byref(my), ctypes.byref(mw),
                                           ctypes.c_void_p(w_scale.data_ptr()), base_scale, ctypes.byref(cfg),
                                           ctypes.byref(mo), st, _stream(stream)))
    return y_out


def ffn_gelu(x_t, x_prev, y1_prev, w1, w1_scale, h_t, h_prev, y2_prev, w2, w2_scale, base_scale: float,
             ws1: Workspace, ws2: Workspace, *, t0: int = 0, force_bits: int = 0, flags1: int = 0, flags2: int = 0,
             debug1=(None, None), debug2=(None, None), stream=None):
    """dstar_fmdq_ffn_gelu: layer 1, H_t = GELU(Y1_t) from its epilogue, layer 2 on
    (H_t, H_{t-1}); y1_prev, y2_prev updated in place, h_t written, h_prev
    refreshed.  debugN = (codes, acc) device buffers of layer N, or None."""
    c1 = _cfg(ws1, t0, force_bits, flags1, *debug1)
    c2 = _cfg(ws2, t0, force_bits, flags2, *debug2)
    m = [mat(t) for t in (x_t, x_prev, y1_prev, w1, h_t, h_prev, y2_prev, w2)]
    _check(lib().dstar_fmdq_ffn_gelu(*(ctypes.byref(v) for v in m[:4]), ctypes.c_void_p(w1_scale.data_ptr()),
                                     *(ctypes.byref(v) for v in m[4:]), ctypes.c_void_p(w2_scale.data_ptr()),
                                     base_scale, ctypes.byref(c1), ctypes.byref(c2), _stream(stream)))
    return y2_prev


class SarAttention:
    """Sparse attention reuse with INT8 FMDQ operands (dstar_sar_attention):
    `heads` problems of `seq` tokens and `head_dim` channels, a host block mask
    [seq/128 x seq/128] (nonzero = kept), its caller-owned workspace."""

    def __init__(self, heads: int, seq: int, head_dim: int, block_mask, scores_scale: float, base_q: float,
                 base_p: float, device="cuda", stream=None):
        import numpy as np
        self.heads, self.seq, self.head_dim = heads, seq, head_dim
        self.mask = np.ascontiguousarray(block_mask, dtype=np.uint8)
        n = ctypes.c_size_t()
        _check(lib().dstar_sar_workspace_size(heads, seq, head_dim, ctypes.byref(n)))
        self.nbytes = n.value
        buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
        off = (-buf.data_ptr()) % 256
        self.buf = buf[off:off + self.nbytes]
        self.cfg = SarCfg(heads, seq, head_dim, self.mask.ctypes.data_as(ctypes.c_void_p), scores_scale, base_q,
                          base_p, ctypes.c_void_p(self.buf.data_ptr()), self.nbytes)
        self.layout = SarLayout()
        _check(lib().dstar_sar_workspace_layout(heads, seq, head_dim, ctypes.byref(self.layout)))
        _check(lib().dstar_sar_workspace_init(ctypes.byref(self.cfg), _stream(stream)))

    def __call__(self, q, k, v, out, reuse: bool = False, stream=None):
        mq, mk, mv, mo = mat(q), mat(k), mat(v), mat(out)
        _check(lib().dstar_sar_attention(ctypes.byref(mq), ctypes.byref(mk), ctypes.byref(mv), ctypes.byref(self.cfg),
                                         int(bool(reuse)), ctypes.byref(mo), _stream(stream)))
        return out

    def status(self, stream=None) -> int:
        s = ctypes.c_uint32()
        _check(lib().dstar_sar_status(ctypes.byref(self.cfg), _stream(stream), ctypes.byref(s)))
        return s.value

    def section(self, name: str, count: int, dtype):
        off = getattr(self.layout, name)
        nb = count * torch.tensor([], dtype=dtype).element_size()
        return self.buf[off:off + nb].view(dtype)

    def fmdq_sections(self, which: str) -> dict:
        """The FMDQ workspace sections of P ('p') or of Q ('q')."""
        R = self.heads * self.seq
        K = self.seq if which == "p" else self.head_dim
        off = getattr(self.layout, "ws_" + which)
        ws = Workspace.__new__(Workspace)
        ws.M, ws.K, ws.nbytes = R, K, workspace_size(R, K)
        ws.buf = self.buf[off:off + ws.nbytes]
        return ws.sections(R, K)


def quantize(x_t, x_prev, base_scale: float, ws: Workspace, *, t0: int = 0, force_bits: int = 0, flags: int = 0,
             debug_codes=None, stream=None):
    """dstar_fmdq_quantize: steps 1-4 into the workspace (and x_prev refresh)."""
    cfg = _cfg(ws, t0, force_bits, flags, debug_codes, None)
    mx, mp = mat(x_t), mat(x_prev)
    _check(lib().dstar_fmdq_quantize(ctypes.byref(mx), ctypes.byref(mp), base_scale, ctypes.byref(cfg),
                                     _stream(stream)))


def slice_gemm(w_q, w_scale, y_prev, base_scale: float, ws: Workspace, *, flags: int = 0, y_out=None,
               debug_acc=None, stream=None):
    """dstar_fmdq_slice_gemm: step 5 and the epilogue from the workspace; returns y_out."""
    if y_out is None:
        y_out = y_prev
    cfg = _cfg(ws, 0, 0, flags, None, debug_acc)
    mw, my, mo = mat(w_q), mat(y_prev), mat(y_out)
    _check(lib().dstar_fmdq_slice_gemm(ctypes.byref(mw), ctypes.c_void_p(w_scale.data_ptr()), ctypes.byref(my),
                                       base_scale, ctypes.byref(cfg), ctypes.byref(mo), _stream(stream)))
    return y_out


def status(ws: Workspace, stream=None) -> int:
    """Read and clear the workspace's sticky status word (synchronises the stream)."""
    s = ctypes.c_uint32()
    _check(lib().dstar_fmdq_status(ctypes.c_void_p(ws.ptr), _stream(stream), ctypes.byref(s)))
    return s.value


def gemm_tile(M: int, N: int, K: int, out_bf16: bool) -> tuple[int, int, bool]:
    """(rows, columns, CTA pair) of the slice GEMM's output tiles for an M x N output with K channels."""
    bm, bn, pair = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    _check(lib().dstar_fmdq_gemm_tile(ctypes.c_int64(M), ctypes.c_int64(N), ctypes.c_int64(K), int(bool(out_bf16)),
                                      ctypes.byref(bm), ctypes.byref(bn), ctypes.byref(pair)))
    return bm.value, bn.value, bool(pair.value)


def selftest_div(b: torch.Tensor, e_lo: int, e_hi: int, stream=None) -> int:
    """dstar_fmdq_selftest_div: how many quotients a / b[i] of the dynamic-base
    division differ from __fdiv_rn over all significands of a in [2^e_lo, 2^(e_hi+1))."""
    assert b.is_cuda and b.dtype == torch.float32 and b.is_contiguous()
    count = torch.zeros(1, dtype=torch.int64, device=b.device)
    _check(lib().dstar_fmdq_selftest_div(ctypes.c_void_p(b.data_ptr()), int(b.numel()), int(e_lo), int(e_hi),
                                         ctypes.c_void_p(count.data_ptr()), _stream(stream)))
    return int(count.item())


def selftest_wait(ws: Workspace, limit_us: int, stream=None):
    _check(lib().dstar_fmdq_selftest_wait(ctypes.c_void_p(ws.ptr), limit_us, _stream(stream)))


def version() -> int:
    return lib().dstar_fmdq_version()
