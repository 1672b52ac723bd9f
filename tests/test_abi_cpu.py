"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function include/*.h declares, report
workspace sizes, and reject bad arguments on the host before touching a
device.
"""
import ctypes
import glob
import os
import re

import pytest

from differential_quantized_gemm_b200 import _native as nat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from differential_quantized_gemm_b200 import build
    build.build()
    return nat.lib()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[\w\s\*]+?\b(dstar_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 11, names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert set(names) == set(nat.EXPORTED)


def test_version_and_strings(L):
    assert nat.version() == 2
    assert L.dstar_fmdq_error_string(-1) == b"invalid argument"
    assert L.dstar_fmdq_error_string(0) == b"ok"


def test_workspace_layout_consistent(L):
    for M, K in [(256, 384), (2048, 1152), (2048, 4608), (16384, 4608), (16, 32)]:
        lay = nat.workspace_layout(M, K)
        T = M // 16
        assert lay.total == nat.workspace_size(M, K)
        assert lay.record_cap == 4 * K
        assert lay.mask_words == ((K + 127) // 128 + 31) // 32
        offs = [lay.status, lay.plane0, lay.plane1, lay.fpot, lay.bits, lay.g_ref, lay.planes, lay.count,
                lay.mask1, lay.records]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert lay.plane1 - lay.plane0 >= M * K and lay.records + T * 4 * K * 8 <= lay.total
        # the dynamic base word sits in the header, after the status word
        assert lay.status + 4 <= lay.dyn_base and lay.dyn_base + 4 <= lay.plane0 and lay.dyn_base % 4 == 0


def _fake_mat(rows, cols, dtype, ptr=0x100000, ld=None):
    return nat.DstarMat(ptr, dtype, 0, rows, cols, cols if ld is None else ld)


def _call_linear(M=64, K=128, N=64, x_dtype=nat.BF16, base=0.0625, ws_bytes=None, cfg_mut=None, **mats):
    x_t = mats.get("x_t", _fake_mat(M, K, x_dtype, 0x100000))
    x_p = mats.get("x_prev", _fake_mat(M, K, x_dtype, 0x200000))
    y_p = mats.get("y_prev", _fake_mat(M, N, nat.BF16, 0x300000))
    w = mats.get("w_q", _fake_mat(N, K, nat.I8, 0x400000))
    y_o = mats.get("y_out", y_p)
    need = nat.workspace_size(M, K) if M % 16 == 0 and 0 < K <= nat.K_MAX else 1 << 20
    cfg = nat.TileCfg(16, 0, 0, 0, ctypes.c_void_p(0x10000000), need if ws_bytes is None else ws_bytes, None, None)
    if cfg_mut:
        cfg_mut(cfg)
    P = lambda m: ctypes.byref(m) if m is not None else None  # noqa: E731
    return nat.lib().dstar_fmdq_linear(P(x_t), P(x_p), P(y_p), P(w), ctypes.c_void_p(0x500000), base,
                                       ctypes.byref(cfg), P(y_o), None)


@pytest.mark.parametrize("case,code", [
    ("M not multiple of 16", -1),
    ("K not multiple of 32", -1),
    ("K too large", -1),
    ("base not power of two", -1),
    ("base out of range", -1),
    ("negative base", -1),
    ("workspace too small", -2),
    ("workspace misaligned", -2),
    ("bad force_bits", -1),
    ("bad tile", -1),
    ("unknown flag", -1),
    ("dtype mismatch", -1),
    ("y partial overlap", -1),
    ("misaligned x", -1),
    ("w not int8", -1),
    ("N not multiple of 16", -1),
    ("null x_t", -1),
])
def test_invalid_arguments_rejected_on_host(L, case, code):
    if case == "M not multiple of 16":
        rc = _call_linear(M=40)
    elif case == "K not multiple of 32":
        rc = _call_linear(K=100)
    elif case == "K too large":
        rc = _call_linear(K=nat.K_MAX + 32)
    elif case == "base not power of two":
        rc = _call_linear(base=0.1)
    elif case == "base out of range":
        rc = _call_linear(base=2.0 ** -40)
    elif case == "negative base":
        rc = _call_linear(base=-0.0625)
    elif case == "workspace too small":
        rc = _call_linear(ws_bytes=1024)
    elif case == "workspace misaligned":
        rc = _call_linear(cfg_mut=lambda c: setattr(c, "workspace", 0x10000010))
    elif case == "bad force_bits":
        rc = _call_linear(cfg_mut=lambda c: setattr(c, "force_bits", 3))
    elif case == "bad tile":
        rc = _call_linear(cfg_mut=lambda c: setattr(c, "tile_tokens", 32))
    elif case == "unknown flag":
        rc = _call_linear(cfg_mut=lambda c: setattr(c, "flags", 0x80))
    elif case == "dtype mismatch":
        rc = _call_linear(x_prev=_fake_mat(64, 128, nat.F32, 0x200000))
    elif case == "y partial overlap":
        rc = _call_linear(y_out=_fake_mat(64, 64, nat.BF16, 0x300000 + 64))
    elif case == "misaligned x":
        rc = _call_linear(x_t=_fake_mat(64, 128, nat.BF16, 0x100008))
    elif case == "w not int8":
        rc = _call_linear(w_q=_fake_mat(64, 128, nat.BF16, 0x400000))
    elif case == "N not multiple of 16":
        rc = _call_linear(N=40)
    elif case == "null x_t":
        rc = nat.lib().dstar_fmdq_linear(None, None, None, None, None, 1.0, None, None, None)
    assert rc == code, (case, rc, nat.lib().dstar_fmdq_last_error())
    assert nat.lib().dstar_fmdq_last_error()  # a reason is given


def test_empty_batch_is_noop(L):
    # M == 0: valid, nothing enqueued, no device needed
    assert _call_linear(M=0) == 0


def test_python_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(nat, "_lib", None)
    monkeypatch.setattr(nat, "LIB_PATH", "/nonexistent/libdstar_fmdq.so")
    with pytest.raises(nat.DstarError, match="not built"):
        nat.lib()
