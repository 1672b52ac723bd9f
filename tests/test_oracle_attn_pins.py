"""Pins of the oracle's attention path: sparse attention reuse (DSTAR section
3.2) with INT8 FMDQ operands (section 4.3, "Attention Operation").  The
per-row int8 rule against element-wise numpy arithmetic, the block-masked
softmax against a numpy softmax of the kept entries and its invariants, and
the whole head against a plain fp64 attention within the quantization error.
CPU only.
"""
import numpy as np
import pytest


def test_quant_rows_elementwise(orc):
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((24, 40)) * rng.uniform(0.01, 10, (24, 1))).astype(np.float32)
    x[5] = 0.0
    q, sc = orc.quant_rows(x)
    for r in range(24):
        mx = np.float32(np.abs(x[r]).max())
        s = np.float32(mx / np.float32(127.0))
        assert sc[r] == s
        for c in range(40):
            want = 0 if mx == 0 else int(np.rint(np.float32(x[r, c]) / s))  # rint: ties to even
            assert q[r, c] == want
    assert np.abs(q.astype(int)).max() <= 127
    big = np.abs(x).argmax(axis=1)
    nz = np.abs(x).max(axis=1) > 0
    assert (np.abs(q[np.arange(24), big])[nz] == 127).all()
    err = np.abs(q.astype(np.float64) * sc[:, None] - x)
    assert (err <= sc[:, None] * 0.5 * (1 + 1e-5) + 1e-12).all()


def _mask(nb, seed, keep=0.6):
    rng = np.random.default_rng(seed)
    m = (rng.random((nb, nb)) < keep).astype(np.uint8)
    np.fill_diagonal(m, 1)
    return m


def test_masked_softmax_against_numpy(orc):
    rng = np.random.default_rng(1)
    blk, nb = 8, 5
    s = (rng.standard_normal((blk * nb, blk * nb)) * 3).astype(np.float32)
    m = _mask(nb, 2)
    p = orc.masked_softmax(s, m, blk)
    keep = np.kron(m, np.ones((blk, blk), np.uint8)).astype(bool)
    for r in range(s.shape[0]):
        e = np.exp(s[r, keep[r]].astype(np.float64) - s[r, keep[r]].astype(np.float64).max())
        assert np.array_equal(p[r, keep[r]], (e / e.sum()).astype(np.float32))
    assert (p[~keep] == 0).all()
    assert np.allclose(p.astype(np.float64).sum(axis=1), 1.0, atol=1e-6)
    # shift invariance (up to the fp32 rounding of the shifted scores)
    p2 = orc.masked_softmax((s + np.float32(4.0)).astype(np.float32), m, blk)
    assert np.allclose(p2, p, rtol=1e-5, atol=1e-7)


def test_head_against_plain_fp64_attention(orc):
    """All blocks kept: the INT8 FMDQ head is within the quantization error of
    softmax(Q K^T / sqrt d) V in fp64 (a transposed operand or a lost scale
    would be far outside)."""
    rng = np.random.default_rng(3)
    S, d, blk = 64, 32, 16
    q = rng.standard_normal((S, d)).astype(np.float32)
    k = rng.standard_normal((S, d)).astype(np.float32)
    v = rng.standard_normal((S, d)).astype(np.float32)
    mask = np.ones((S // blk, S // blk), np.uint8)
    scale = np.float32(1.0 / np.sqrt(d))
    r = orc.sar_attention(q, k, v, mask, blk, -4, -6, scale)
    sc = (q.astype(np.float64) @ k.astype(np.float64).T) * float(scale)
    assert np.abs(r["scores"] - sc).max() < 0.05 * np.abs(sc).max()
    e = np.exp(sc - sc.max(axis=1, keepdims=True))
    ref = (e / e.sum(axis=1, keepdims=True)) @ v.astype(np.float64)
    assert np.abs(r["out"] - ref).max() < 0.05 * np.abs(ref).max()
    assert np.abs(r["out"] - ref).mean() < 0.05 * np.abs(ref).mean()


def test_reuse_step_uses_the_cached_p(orc):
    rng = np.random.default_rng(4)
    S, d, blk = 48, 32, 16
    q, k, v = (rng.standard_normal((S, d)).astype(np.float32) for _ in range(3))
    mask = _mask(S // blk, 5)
    cached = orc.sar_attention(q, k, v, mask, blk, -4, -6, np.float32(1 / np.sqrt(d)))
    v2 = rng.standard_normal((S, d)).astype(np.float32)
    reused = orc.sar_attention(q * 7, k * 7, v2, mask, blk, -4, -6, np.float32(1 / np.sqrt(d)),
                               p_cached=cached["qP"])
    fresh_p = orc.sar_attention(q, k, v2, mask, blk, -4, -6, np.float32(1 / np.sqrt(d)))
    assert np.array_equal(reused["out"], fresh_p["out"])  # Q and K of the reused step are never read
    assert "scores" not in reused
    # pruned blocks stay pruned in the cached P
    keep = np.kron(mask, np.ones((blk, blk), np.uint8)).astype(bool)
    assert (cached["p"][~keep] == 0).all() and not cached["qP"].codes[~keep].any()
