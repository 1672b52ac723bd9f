"""Seeded synthetic inputs for the FMDQ differential linear layer.

This module holds input recipes only: random activations, differentials,
int8 weights with per-output-channel scales and the cached previous output.
It contains none of the method's arithmetic; both the CUDA path and the CPU
oracle receive the same bytes from it.

The trained DiT checkpoints and COCO/FETV prompts of the paper's evaluation
(section 5.1) are not available, so each workload below is a synthetic
stand-in with the shapes of the paper's models (DiT-XL/2, PixArt-Sigma,
Latte) and a differential distribution chosen to produce the bit-width mixes
the paper describes (section 3.1: first and last steps change most sharply;
Fig. 14: 2-8 bit mixes).

Arrays are numpy; bf16 tensors are carried as uint16 bit patterns (rounded to
nearest-even from fp32).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest, ties to even."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class LayerSpec:
    name: str
    M: int
    K: int
    N: int
    dtype: str  # "f32" or "bf16"
    lb: int     # base scale = 2^lb
    t0: int = 0
    force_bits: int = 0


@dataclass
class LayerInputs:
    spec: LayerSpec
    x_t: np.ndarray      # [M x K] float32 values, or uint16 bf16 bits
    x_prev: np.ndarray   # same dtype as x_t
    y_prev: np.ndarray   # [M x N] same dtype convention
    w_q: np.ndarray      # [N x K] int8 in [-127, 127]
    w_scale: np.ndarray  # [N] float32

    def as_f32(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        return bf16_bits_to_f32(a) if self.spec.dtype == "bf16" else a


# ------------------------------------------------------------------ configs

CONFIG_NAMES = {
    1: "tiny single linear 256x384->384 fp32",
    2: "DiT-XL/2 256px FFN pair, batch 8x256 tokens, bf16",
    3: "PixArt 1024px layer, batch 2x4096 tokens, bf16",
    4: "Latte video FFN, batch 4x16 frames x256 tokens, bf16",
    5: "28-layer DiT-XL FFN stack timestep sweep, batch 8x1024 tokens, bf16",
}


def config_layers(cfg: int) -> list[LayerSpec]:
    if cfg == 1:
        return [LayerSpec("linear", 256, 384, 384, "f32", -10)]
    if cfg == 2:
        return [LayerSpec("ffn_up", 2048, 1152, 4608, "bf16", -4),
                LayerSpec("ffn_down", 2048, 4608, 1152, "bf16", -4)]
    if cfg == 3:
        return [LayerSpec("qkv", 8192, 1152, 3456, "bf16", -4),
                LayerSpec("out_proj", 8192, 1152, 1152, "bf16", -4),
                LayerSpec("ffn_up", 8192, 1152, 4608, "bf16", -4),
                LayerSpec("ffn_down", 8192, 4608, 1152, "bf16", -4)]
    if cfg == 4:
        return [LayerSpec("ffn_up", 16384, 1152, 4608, "bf16", -4),
                LayerSpec("ffn_down", 16384, 4608, 1152, "bf16", -4)]
    if cfg == 5:
        return [LayerSpec(f"l{i}_{kind}", 8192, K, N, "bf16", -4)
                for i in range(28) for kind, K, N in (("up", 1152, 4608), ("down", 4608, 1152))]
    raise ValueError(cfg)


def sweep_sigma(step: int, steps: int = 50) -> float:
    """U-shaped differential scale of the timestep sweep: log-linear from 0.3 at
    step 0 down to 0.01 at the middle step, then up to 0.1 at the last step."""
    mid = steps // 2
    if step <= mid:
        a = step / mid
        return math.exp((1 - a) * math.log(0.3) + a * math.log(0.01))
    a = (step - mid) / (steps - 1 - mid)
    return math.exp((1 - a) * math.log(0.01) + a * math.log(0.1))


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _weights(rng, K, N):
    w_q = rng.integers(-127, 128, size=(N, K), dtype=np.int16).astype(np.int8)
    w_scale = rng.uniform(0.001, 0.01, size=N).astype(np.float32)
    return w_q, w_scale


def layer_weights(cfg: int, layer: int, seed: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """The int8 weights and per-output-channel scales make_layer draws for
    (cfg, layer), without drawing the activations."""
    spec = config_layers(cfg)[layer]
    return _weights(_rng(cfg if seed is None else seed, layer, 101), spec.K, spec.N)


def _dx(cfg: int, spec: LayerSpec, rng, sigma: float | None) -> np.ndarray:
    M, K = spec.M, spec.K
    if cfg == 1:
        return (0.05 * rng.standard_normal((M, K))).astype(np.float32)
    if cfg == 2:
        dx = 0.03 * rng.standard_normal((M, K), dtype=np.float32)
        hit = rng.random((M, K), dtype=np.float32) < 0.01
        dx[hit] = 0.5 * rng.standard_normal(int(hit.sum()), dtype=np.float32)
        return dx
    if cfg == 3:
        T = M // 16
        sig = np.exp(rng.uniform(math.log(1e-3), math.log(1.0), size=T)).astype(np.float32)
        return rng.standard_normal((M, K), dtype=np.float32) * np.repeat(sig, 16)[:, None]
    if cfg == 4:
        # tokens ordered (batch, frame, patch); 256 patches per frame at full size,
        # fewer for small test cases, always whole 16-token tiles per frame
        F = 16
        Pn = min(256, max(16, (M // F) // 16 * 16))
        B = M // (F * Pn)
        assert B * F * Pn == M, "video workload needs M = batch x 16 frames x patches"
        z = rng.standard_normal((B, F, Pn, K), dtype=np.float32)
        e = np.empty_like(z)
        e[:, 0] = 0.05 * z[:, 0]
        c = np.float32(0.05 * math.sqrt(1 - 0.81))
        for f in range(1, F):
            e[:, f] = np.float32(0.9) * e[:, f - 1] + c * z[:, f]
        dx = e.reshape(M, K)
        rows = rng.random(M) < 0.05
        dx[rows] = 0.5 * rng.standard_normal((int(rows.sum()), K), dtype=np.float32)
        return dx
    if cfg == 5:
        s = 0.03 if sigma is None else sigma
        return (s * rng.standard_normal((M, K), dtype=np.float32))
    raise ValueError(cfg)


def make_layer(cfg: int, layer: int = 0, step: int = 0, force_bits: int = 0, seed: int | None = None,
               M: int | None = None) -> LayerInputs:
    """Inputs of one differential linear call.

    cfg, layer, step and seed select the deterministic draw; M may shrink the
    token count (a multiple of 16, keeping whole frames for the video config)
    for small test cases with the same value distributions.
    """
    spec = config_layers(cfg)[layer]
    if M is not None:
        spec = LayerSpec(spec.name, M, spec.K, spec.N, spec.dtype, spec.lb, spec.t0, spec.force_bits)
    if force_bits:
        spec.force_bits = force_bits
    base_seed = cfg if seed is None else seed
    rng_w = _rng(base_seed, layer, 101)
    rng_x = _rng(base_seed, layer, 202)
    rng_d = _rng(base_seed, layer, 303, step)

    w_q, w_scale = _weights(rng_w, spec.K, spec.N)
    x_prev = rng_x.standard_normal((spec.M, spec.K), dtype=np.float32)
    if cfg == 2:
        nout = int(round(0.02 * spec.K))
        ch = rng_x.choice(spec.K, size=nout, replace=False)
        x_prev[:, ch] *= 8.0
    sigma = sweep_sigma(step) if cfg == 5 else None
    if cfg == 5 and force_bits:
        sigma = 0.03
    dx = _dx(cfg, spec, rng_d, sigma)

    # step-0 dense initialisation of the cached output, Y_{t-1} = X_{t-1} W_deq
    w_deq_t = w_q.astype(np.float32).T * w_scale[None, :]
    if spec.dtype == "bf16":
        xp_b = to_bf16_bits(x_prev)
        xp_f = bf16_bits_to_f32(xp_b)
        xt_b = to_bf16_bits(xp_f + dx)
        y = xp_f @ w_deq_t
        return LayerInputs(spec, xt_b, xp_b, to_bf16_bits(y), w_q, w_scale)
    x_t = (x_prev + dx).astype(np.float32)
    y = (x_prev.astype(np.float64) @ w_deq_t.astype(np.float64)).astype(np.float32)
    return LayerInputs(spec, x_t, x_prev, y, w_q, w_scale)


def adversarial_layer(M: int, K: int, N: int, seed: int, spread: int = 24, dtype: str = "bf16",
                      lb: int = -4) -> LayerInputs:
    """A stress input: per sub-channel magnitudes spread over 2^spread, so tiles
    mix every bit width and a wide range of scales (many FPoT groups)."""
    rng = _rng(seed, 7, 7)
    w_q, w_scale = _weights(rng, K, N)
    x_prev = rng.standard_normal((M, K), dtype=np.float32)
    # each tile draws its own spread in [0, spread]: some tiles are narrow, some wide
    tile_spread = rng.uniform(0, spread, size=(M // 16, 1))
    mag = np.exp2(-8 + tile_spread * rng.uniform(0, 1, size=(M // 16, K))).astype(np.float32)
    dx = rng.standard_normal((M, K), dtype=np.float32) * np.repeat(mag, 16, axis=0)
    spec = LayerSpec("adversarial", M, K, N, dtype, lb)
    w_deq_t = w_q.astype(np.float32).T * w_scale[None, :]
    if dtype == "bf16":
        xp_b = to_bf16_bits(x_prev)
        xp_f = bf16_bits_to_f32(xp_b)
        xt_b = to_bf16_bits(xp_f + dx)
        return LayerInputs(spec, xt_b, xp_b, to_bf16_bits(xp_f @ w_deq_t), w_q, w_scale)
    x_t = (x_prev + dx).astype(np.float32)
    return LayerInputs(spec, x_t, x_prev, (x_prev @ w_deq_t).astype(np.float32), w_q, w_scale)


class SweepChain:
    """Consecutive calls of one layer of the timestep sweep with the caches
    carried: X at each listed step is the previous X plus sigma_t * N(0, 1)
    (rounded to bf16), starting from X_{-1} ~ N(0, 1); the cached output
    starts from the dense product and is carried by each side itself."""

    def __init__(self, layer: int, steps: list[int], M: int = 8192, force_bits: int = 0):
        self.layer, self.step_list, self.force_bits = layer, list(steps), force_bits
        spec = config_layers(5)[layer]
        self.spec = LayerSpec(spec.name, M, spec.K, spec.N, "bf16", spec.lb, spec.t0, force_bits)

    def steps(self):
        spec = self.spec
        rng_w = _rng(5, self.layer, 101)
        rng_x = _rng(5, self.layer, 202)
        w_q, w_scale = _weights(rng_w, spec.K, spec.N)
        x = to_bf16_bits(rng_x.standard_normal((spec.M, spec.K), dtype=np.float32))
        xf = bf16_bits_to_f32(x)
        y = to_bf16_bits(xf @ (w_q.astype(np.float32).T * w_scale[None, :]))
        for s in self.step_list:
            sig = 0.03 if self.force_bits else sweep_sigma(s)
            z = _rng(5, self.layer, 303, s).standard_normal((spec.M, spec.K), dtype=np.float32)
            x_new = to_bf16_bits(bf16_bits_to_f32(x) + np.float32(sig) * z)
            yield LayerInputs(spec, x_new, x, y, w_q, w_scale)
            x = x_new


def sweep_chain(layer: int, steps: list[int], M: int = 8192, force_bits: int = 0) -> SweepChain:
    return SweepChain(layer, steps, M, force_bits)


def attention_inputs(heads: int, seq: int, head_dim: int, pad_to: int, seed: int, keep: float = 0.5):
    """Seeded Q, K, V for `heads` attention problems of `seq` tokens: N(0, 1)
    in the first head_dim channels, zero padding up to pad_to (bf16 bit
    patterns, [heads*seq x pad_to]); V of the next step (V plus a 0.05 N(0, 1)
    change); and a block mask [seq/128 x seq/128] that keeps every diagonal
    block and each other block with probability `keep` (the pages' masks come
    from profiling trained models, which are not available)."""
    rng = _rng(seed, 909)
    R = heads * seq

    def draw():
        x = np.zeros((R, pad_to), np.float32)
        x[:, :head_dim] = rng.standard_normal((R, head_dim), dtype=np.float32)
        return x

    q, k, v = draw(), draw(), draw()
    v2 = v.copy()
    v2[:, :head_dim] += 0.05 * rng.standard_normal((R, head_dim), dtype=np.float32)
    nb = seq // 128
    mask = (rng.random((nb, nb)) < keep).astype(np.uint8)
    np.fill_diagonal(mask, 1)
    return to_bf16_bits(q), to_bf16_bits(k), to_bf16_bits(v), to_bf16_bits(v2), mask
