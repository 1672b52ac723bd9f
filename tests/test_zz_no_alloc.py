"""dstar_fmdq_linear_noalloc: the differential linear for callers that cannot
allocate device memory (plug-in layers and custom operators that are handed
only their input and output buffers, loops that must not call cudaMalloc,
hosts whose allocator owns all device memory).  It keeps its scratch in a
static device array of the library instead of a caller-made workspace.

The GPU test calls it through the C ABI twice in a row, with the caches
carried from one call to the next, and checks each result against
dstar_fmdq_linear with a workspace on separate copies of the same buffers:
both run the same kernels, so Y_t must agree bit for bit.  It must pass in a
fresh process (the first call in a context clears the array's status word)
and after the other tests.  This file is named so that pytest collects it
last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from differential_quantized_gemm_b200 import _native as nat
from differential_quantized_gemm_b200 import synth
from gpu_helpers import assert_y_close, dev_to_f32, to_dev


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    """A shape whose scratch exceeds the array is refused on the host with a
    WORKSPACE error that names the limit; nothing touches a device."""
    L = nat.lib()
    M, K = 8192, 4608  # about 156 MB of scratch
    assert nat.workspace_size(M, K) > nat.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    x = nat.DstarMat(fake, nat.BF16, 0, M, K, K)
    cfg = nat.TileCfg(nat.TILE, 0, 0, 0, None, 0, None, None)
    rc = L.dstar_fmdq_linear_noalloc(ctypes.byref(x), ctypes.byref(x), None, None, None, 1.0, ctypes.byref(cfg),
                                     None, None, None)
    assert rc == -2
    msg = L.dstar_fmdq_last_error().decode()
    assert str(nat.NOALLOC_SCRATCH_BYTES) in msg and "static scratch" in msg, msg
    # a caller-supplied workspace is refused too: this entry point has its own
    cfg_ws = nat.TileCfg(nat.TILE, 0, 0, 0, fake, 1 << 20, None, None)
    x_small = nat.DstarMat(fake, nat.BF16, 0, 64, 128, 128)
    rc = L.dstar_fmdq_linear_noalloc(ctypes.byref(x_small), ctypes.byref(x_small), None, None, None, 1.0,
                                     ctypes.byref(cfg_ws), None, None, None)
    assert rc == -1


@pytest.mark.gpu
def test_noalloc_matches_workspace_path_on_two_calls_in_a_row():
    torch.cuda.set_device(0)
    M = 512  # DiT-XL/2 FFN up-projection (1152 -> 4608), 512 tokens, bf16
    chain = synth.sweep_chain(0, steps=[10, 11], M=M)
    spec = chain.spec
    assert nat.workspace_size(M, spec.K) <= nat.NOALLOC_SCRATCH_BYTES
    ws = nat.Workspace(M, spec.K)
    ref = alt = None
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call, inp in enumerate(chain.steps()):
        if ref is None:
            ref = to_dev(inp)  # workspace path: dstar_fmdq_linear
            alt = {k: v.clone() for k, v in ref.items()}  # static-scratch path
        else:
            x_t = torch.from_numpy(inp.x_t).view(torch.bfloat16).cuda()
            ref["x_t"], alt["x_t"] = x_t, x_t.clone()
        base = 2.0 ** spec.lb
        y_ref = nat.linear(ref["x_t"], ref["x_prev"], ref["y_prev"], ref["w_q"], ref["w_scale"], base, ws,
                           t0=spec.t0, force_bits=spec.force_bits)
        status.fill_(-1)
        y_alt = nat.linear_noalloc(alt["x_t"], alt["x_prev"], alt["y_prev"], alt["w_q"], alt["w_scale"], base,
                                   t0=spec.t0, force_bits=spec.force_bits, status_out=status)
        torch.cuda.synchronize()
        assert nat.status(ws) == 0
        assert int(status.item()) == 0, f"call {call}: static-scratch status {int(status.item())}"
        y_r, y_a = dev_to_f32(y_ref), dev_to_f32(y_alt)
        assert np.isfinite(y_a).all()
        assert np.abs(y_r).max() > 0, "the reference output is all zero: the comparison would be empty"
        # the same kernels on the same inputs: Y_t must agree bit for bit;
        # assert_y_close runs first only for the error summary it prints
        assert_y_close(y_a, y_r)
        assert torch.equal(y_alt, y_ref), f"call {call}: Y_t differs from the workspace path"
        # the caches the next call reads: X_{t-1} refreshed the same way
        assert torch.equal(alt["x_prev"], ref["x_prev"]), f"call {call}: x_prev refresh differs"
