"""GPU parity of the chained FFN pair with the GELU fused into layer 1's
epilogue (DSTAR section 4.3 "Operator Mapping") against the oracle's pair,
over consecutive steps with every cache carried on both sides:

- layer 1 (codes, widths, FPoT, g_ref, encoded stream, int64 accumulators)
  bit-exact, Y1_t within the tolerance;
- H_t = GELU(Y1_t) within one bf16 ulp of the oracle's fp64 GELU everywhere
  and equal to it almost everywhere (the library's table is filled in fp64
  with CUDA's erfc, the oracle's with the C library's: they round to the same
  bf16 value except next to a rounding boundary);
- layer 2: the GPU's and the oracle's inputs differ wherever their H differ,
  so its integer outputs are compared on every sub-channel (and every tile)
  whose inputs agree bit for bit, Y2_t within the tolerance everywhere.
"""
import numpy as np
import pytest
import torch

import oracle
from differential_quantized_gemm_b200 import _native as nat
from differential_quantized_gemm_b200 import synth

from gpu_helpers import Y_MAX_ABS, Y_REL_L2, assert_y_close, y_errors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _build():
    from differential_quantized_gemm_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(oracle.f32_to_bf16(a))).view(torch.bfloat16).cuda()


def _f32(t):
    return t.float().cpu().numpy()


def _ordered(a):
    """fp32 bit patterns mapped to integers in the order of the values (both zeros to 0)."""
    b = a.view(np.int32).astype(np.int64)
    return np.where(b < 0, -(b & 0x7FFFFFFF), b)


def _records(ws, M, K):
    rec = ws.sections(M, K)["records"].cpu().numpy().view(np.uint32)
    return rec[:, :, 0], rec[:, :, 1]


def _pair_inputs(cfg, M):
    """Layer 1 of the workload's FFN pair and the second layer's weights; the
    caches start from the dense state: H_{t-1} = GELU(Y1_{t-1}),
    Y2_{t-1} = H_{t-1} W2_deq (fp64, rounded to bf16)."""
    up = synth.make_layer(cfg, 0, M=M)
    w2, ws2 = synth.layer_weights(cfg, 1)
    y1p = up.as_f32("y_prev")
    hp = oracle.gelu(y1p, True)
    y2p = oracle.bf16_to_f32(oracle.f32_to_bf16(
        (hp.astype(np.float64) @ (w2.astype(np.float64).T * ws2.astype(np.float64)[None, :])).astype(np.float32)))
    return up, w2, ws2, y1p, hp, y2p


def _chain(cfg, M, steps, flags=0):
    up, w2, ws2, y1p, hp, y2p = _pair_inputs(cfg, M)
    s = up.spec
    K1, N1, N2 = s.K, s.N, w2.shape[0]
    d = dict(x_prev=_bf(up.as_f32("x_prev")), y1=_bf(y1p), h_prev=_bf(hp), y2=_bf(y2p),
             w1=torch.from_numpy(up.w_q).cuda(), s1=torch.from_numpy(up.w_scale).cuda(),
             w2=torch.from_numpy(w2).cuda(), s2=torch.from_numpy(ws2).cuda())
    h_t = torch.empty(M, N1, dtype=torch.bfloat16, device="cuda")
    ws1, wsb = nat.Workspace(M, K1), nat.Workspace(M, N1)
    x_prev_o, y1_o, h_prev_o, y2_o = up.as_f32("x_prev"), y1p, hp, y2p
    x = up.as_f32("x_t")
    h_prev_gpu = hp  # both sides start from the same H_{t-1}
    rng = np.random.default_rng(cfg)
    compared_sub = total_sub = compared_tiles = 0
    for step in range(steps):
        if step > 0:  # the next step's input: a new differential on the current X
            x = oracle.bf16_to_f32(oracle.f32_to_bf16(x + 0.03 * rng.standard_normal(x.shape).astype(np.float32)))
        x_t = _bf(x)
        c1 = torch.zeros(M, K1, dtype=torch.int8, device="cuda")
        a1 = torch.zeros(M, N1, dtype=torch.int64, device="cuda")
        c2 = torch.zeros(M, N1, dtype=torch.int8, device="cuda")
        a2 = torch.zeros(M, N2, dtype=torch.int64, device="cuda")
        nat.ffn_gelu(x_t, d["x_prev"], d["y1"], d["w1"], d["s1"], h_t, d["h_prev"], d["y2"], d["w2"], d["s2"],
                     2.0 ** s.lb, ws1, wsb, flags1=flags, flags2=flags, debug1=(c1, a1), debug2=(c2, a2))
        torch.cuda.synchronize()
        assert nat.status(ws1) == 0 and nat.status(wsb) == 0
        q1, acc1, y1, h, q2, acc2, y2 = oracle.ffn_gelu(x, x_prev_o, y1_o, up.w_q, up.w_scale, h_prev_o, y2_o,
                                                        w2, ws2, s.lb)
        # layer 1: everything
        assert np.array_equal(c1.cpu().numpy(), q1.codes)
        sec1 = ws1.sections(M, K1)
        assert np.array_equal(sec1["fpot"].cpu().numpy(), q1.fpot)
        assert np.array_equal(sec1["count"].cpu().numpy(), q1.count)
        assert np.array_equal(a1.cpu().numpy(), acc1)
        assert_y_close(_f32(d["y1"]), y1)
        # H_t: within one bf16 ulp, nearly always equal
        hg = _f32(h_t)
        ulp = np.abs(_ordered(hg) - _ordered(h)) >> 16
        assert ulp.max() <= 1, ulp.max()
        assert (hg == h).mean() > 0.99999, (hg == h).mean()
        # H_{t-1} was refreshed to the GPU's H_t
        assert torch.equal(d["h_prev"], h_t)
        # layer 2: sub-channels whose 16 inputs (H_t and H_{t-1}) agree
        T = M // 16
        same = ((hg == h) & (h_prev_gpu == h_prev_o)).reshape(T, 16, N1).all(axis=1)
        total_sub += same.size
        compared_sub += int(same.sum())
        sec2 = wsb.sections(M, N1)
        codes2 = c2.cpu().numpy().reshape(T, 16, N1)
        assert np.array_equal(codes2.transpose(0, 2, 1)[same], q2.codes.reshape(T, 16, N1).transpose(0, 2, 1)[same])
        assert np.array_equal(sec2["fpot"].cpu().numpy()[same], q2.fpot[same])
        assert np.array_equal(sec2["bits"].cpu().numpy()[same], q2.bits[same])
        tiles = same.all(axis=1)
        compared_tiles += int(tiles.sum())
        rows = np.repeat(tiles, 16)
        assert np.array_equal(sec2["g_ref"].cpu().numpy()[tiles], q2.g_ref[tiles])
        assert np.array_equal(sec2["count"].cpu().numpy()[tiles], q2.count[tiles])
        word, meta = _records(wsb, M, N1)
        for t in np.flatnonzero(tiles):
            n = q2.count[t]
            assert np.array_equal(word[t, :n], q2.rec_word[t, :n])
            assert np.array_equal((meta[t, :n] & 0xFFFF).astype(np.uint16), q2.rec_k[t, :n])
        assert np.array_equal(a2.cpu().numpy()[rows], acc2[rows])
        max_abs, rel, _ = y_errors(_f32(d["y2"]), y2)
        assert max_abs <= Y_MAX_ABS and rel <= Y_REL_L2, (max_abs, rel)
        # both sides carry their own caches into the next step
        h_prev_gpu = hg
        x_prev_o, y1_o, h_prev_o, y2_o = x, y1, h, y2
    assert compared_sub >= 0.99 * total_sub, (compared_sub, total_sub)
    assert compared_tiles > 0
    return compared_sub / total_sub


def test_ffn_gelu_small_two_steps():
    _chain(2, 3 * 128 + 48, steps=2)


@pytest.mark.parametrize("form", [nat.TILE_128x128, nat.TILE_128x256, nat.TILE_PAIR_256x256, nat.TILE_PAIR_256x128])
def test_ffn_gelu_every_tile_form(form):
    """Both layers in one forced tile form: the activation output of layer 1's
    epilogue from single CTAs and from CTA pairs."""
    _chain(2, 3 * 128 + 48, steps=1, flags=nat.tile_flag(form))


def test_ffn_gelu_full_size_latte():
    """The Latte video FFN pair at 16384 tokens."""
    _chain(4, 16384, steps=1)


def test_ffn_gelu_rejects_shared_workspace_and_overlaps():
    up, w2, ws2, y1p, hp, y2p = _pair_inputs(2, 64)
    s = up.spec
    x = _bf(up.as_f32("x_t"))
    xp, y1, h, y2 = _bf(up.as_f32("x_prev")), _bf(y1p), _bf(hp), _bf(y2p)
    w1, s1 = torch.from_numpy(up.w_q).cuda(), torch.from_numpy(up.w_scale).cuda()
    w2t, s2 = torch.from_numpy(w2).cuda(), torch.from_numpy(ws2).cuda()
    ws = nat.Workspace(64, max(s.K, s.N))
    with pytest.raises(nat.DstarError, match="two workspaces"):
        nat.ffn_gelu(x, xp, y1, w1, s1, h.clone(), h, y2, w2t, s2, 2.0 ** s.lb, ws, ws)
    with pytest.raises(nat.DstarError, match="disjoint"):
        nat.ffn_gelu(x, xp, y1, w1, s1, h, h, y2, w2t, s2, 2.0 ** s.lb, nat.Workspace(64, s.K),
                     nat.Workspace(64, s.N))
