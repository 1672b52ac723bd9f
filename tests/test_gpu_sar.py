"""GPU parity of sparse attention reuse with INT8 FMDQ operands (DSTAR
section 3.2 "Sparse Attention Reuse", section 4.3 "Attention Operation")
against the oracle, head by head, through the C ABI (dstar_sar_attention):

- cached step: the int8 keys and values and their scales, every integer output of Q's
  FMDQ (width, FPoT, g_ref, encoded stream) and the scores of every kept
  block bit-exact; the softmax (fp64 on both sides, rounded once to fp32;
  the library exp and the order of the sums may differ in the last fp64
  bit) equal to the oracle's almost everywhere, pruned entries exactly 0;
  P's FMDQ compared on every sub-channel whose 16 probabilities agree bit
  for bit (at least 99.9 % of them); the output within the tolerance;
- reused step: a new V against the same cached P; Q and K are not read.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from differential_quantized_gemm_b200 import _native as nat
from differential_quantized_gemm_b200 import synth

from gpu_helpers import Y_MAX_ABS, Y_REL_L2, y_errors

pytestmark = pytest.mark.gpu

LB_Q, LB_P = -4, -6


@pytest.fixture(scope="module", autouse=True)
def _build():
    from differential_quantized_gemm_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def _run(G, S, dh, d, seed, heads_checked=None, keep=0.5):
    qb, kb, vb, v2b, mask = synth.attention_inputs(G, S, dh, d, seed, keep)
    scale = float(np.float32(1.0 / math.sqrt(dh)))
    att = nat.SarAttention(G, S, d, mask, scale, 2.0 ** LB_Q, 2.0 ** LB_P)
    q, k, v, v2 = _dev(qb), _dev(kb), _dev(vb), _dev(v2b)
    out = torch.empty(G * S, d, dtype=torch.float32, device="cuda")
    att(q, k, v, out)
    torch.cuda.synchronize()
    assert att.status() == 0
    R = G * S
    got = dict(out=out.cpu().numpy().copy(),
               kq=att.section("kq", R * d, torch.int8).view(R, d).cpu().numpy(),
               ks=att.section("ks", R, torch.float32).cpu().numpy(),
               vqt=att.section("vqt", G * d * S, torch.int8).view(G * d, S).cpu().numpy(),
               vs=att.section("vs", G * d, torch.float32).cpu().numpy(),
               scores=att.section("scores", R * S, torch.float32).view(R, S).clone(),  # on the device
               probs=att.section("probs", R * S, torch.float32).view(R, S).clone(),
               sq={n: t.cpu().numpy() for n, t in att.fmdq_sections("q").items() if n != "plane0" and n != "plane1"},
               sp={n: t.cpu().numpy() for n, t in att.fmdq_sections("p").items() if n in ("fpot", "bits", "g_ref",
                                                                                           "count", "records")})
    att(q, k, v2, out, reuse=True)  # reused step: the cached P with the next V
    torch.cuda.synchronize()
    assert att.status() == 0
    got["out2"] = out.cpu().numpy().copy()
    qf, kf, vf, v2f = (synth.bf16_bits_to_f32(a) for a in (qb, kb, vb, v2b))
    keep_el = np.kron(mask, np.ones((128, 128), np.uint8)).astype(bool)
    T = S // 16
    stats = dict(sub=0, sub_equal=0)
    for h in (range(G) if heads_checked is None else heads_checked):
        rows = slice(h * S, (h + 1) * S)
        ref = oracle.sar_attention(qf[rows], kf[rows], vf[rows], mask, 128, LB_Q, LB_P, np.float32(scale))
        # keys: int8 codes and scales (times the score scale)
        assert np.array_equal(got["kq"][rows], ref["kq"])
        assert np.array_equal(got["ks"][rows], (ref["ks"] * np.float32(scale)).astype(np.float32))
        # values: int8 codes per column of the head's V, stored transposed, and their scales
        assert np.array_equal(got["vqt"][h * d:(h + 1) * d], ref["vq"])
        assert np.array_equal(got["vs"][h * d:(h + 1) * d], ref["vs"])
        # Q's FMDQ (every width 8, X_{t-1} = 0)
        tq = slice(h * T, (h + 1) * T)
        for name in ("fpot", "bits", "g_ref", "count"):
            assert np.array_equal(got["sq"][name][tq], getattr(ref["qQ"], name)), name
        rec = got["sq"]["records"][tq].view(np.uint32)
        for t in range(T):
            n = ref["qQ"].count[t]
            assert np.array_equal(rec[t, :n, 0], ref["qQ"].rec_word[t, :n])
        # scores of the kept blocks, bit for bit
        sc = got["scores"][rows].cpu().numpy()
        assert np.array_equal(sc[keep_el], ref["scores"][keep_el])
        # softmax: fp64 on both sides, rounded once to fp32
        pr = got["probs"][rows].cpu().numpy()
        assert (pr[~keep_el] == 0).all()
        assert np.allclose(pr, ref["p"], rtol=2e-7, atol=1e-12)
        assert (pr == ref["p"]).mean() > 0.9999
        # P's FMDQ on sub-channels whose inputs agree exactly
        same = (pr == ref["p"]).reshape(T, 16, S).all(axis=1)
        stats["sub"] += same.size
        stats["sub_equal"] += int(same.sum())
        for name in ("fpot", "bits"):
            assert np.array_equal(got["sp"][name][tq][same], getattr(ref["qP"], name)[same]), name
        # the outputs of both steps
        for key, v_ref in (("out", None), ("out2", v2f[rows])):
            o_ref = ref["out"] if v_ref is None else oracle.sar_attention(
                qf[rows], kf[rows], v_ref, mask, 128, LB_Q, LB_P, np.float32(scale), p_cached=ref["qP"])["out"]
            max_abs, rel, _ = y_errors(got[key][rows], o_ref)
            assert max_abs <= Y_MAX_ABS and rel <= Y_REL_L2, (key, h, max_abs, rel)
    assert stats["sub_equal"] >= 0.999 * stats["sub"], stats
    return got, mask


def test_sar_dit_xl_heads():
    """DiT-XL/2 256px attention: 256 tokens, head dimension 72 padded to 96."""
    got, mask = _run(G=4, S=256, dh=72, d=96, seed=1)


def test_sar_1024_tokens_sparse_mask():
    got, mask = _run(G=2, S=1024, dh=72, d=96, seed=2, keep=0.4)
    assert mask.sum() < mask.size  # some blocks are pruned


def test_sar_pixart_full_size_two_heads_checked():
    """PixArt 1024px attention: 2 x 16 heads of 4096 tokens, the first and last
    head compared in full."""
    _run(G=32, S=4096, dh=72, d=96, seed=3, heads_checked=[0, 31])


def test_sar_rejects_a_mask_row_without_blocks():
    mask = np.ones((2, 2), np.uint8)
    mask[1] = 0
    att = nat.SarAttention(1, 256, 32, mask, 0.125, 2.0 ** LB_Q, 2.0 ** LB_P)
    x = torch.zeros(256, 32, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(256, 32, dtype=torch.float32, device="cuda")
    with pytest.raises(nat.DstarError, match="keeps no block"):
        att(x, x, x, out)
