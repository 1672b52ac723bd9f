"""B200-native (sm_100a) FMDQ differential linear layer.

DSTAR's fine-grained mixed-precision differential quantization of DiT linear
layers: Y_t = Y_{t-1} + dequant(Q(X_t - X_{t-1}) W_q), with per-sub-channel
power-of-two scales, 2/4/6/8-bit widths, 2-bit slices grouped by FPoT and
shift-aligned accumulation on int8 tensor cores.

The computation lives in the CUDA library built from csrc/ (C ABI in
include/dstar_fmdq.h); this package is its Python binding.
"""
from ._native import (  # noqa: F401
    BF16, F32, FLAG_DYNAMIC_BASE, FLAG_NO_XPREV_REFRESH, FLAG_SLICE_PATH, I8, POT_MAX, STATUS_NONFINITE, STATUS_RANGE,
    STATUS_TIMEOUT, TILE, DstarError, Workspace, lib, linear, quantize, selftest_wait, slice_gemm, status,
    version, workspace_layout, workspace_size,
)
