"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and casts them to storage formats; it holds
none of the quantization or GEMM arithmetic.  Everything is generated on the
CPU with ``numpy.random.default_rng(seed)`` and cast to bf16 (round to nearest
even) through torch, so the oracle and the CUDA path read the same bytes.

Shapes follow the Qwen3 family the pages benchmark ("Helion in vLLM"
(24-ai.news), section "Full-model speedups": Qwen3 1.7B / 8B / 32B):
  Qwen3-8B   hidden 4096, intermediate 12288, 32 q heads / 8 kv heads of 128
  Qwen3-32B  hidden 5120, intermediate 25600, 64 q heads / 8 kv heads of 128
"""
from __future__ import annotations

import numpy as np
import torch

QWEN3_8B = dict(hidden=4096, intermediate=12288, q_heads=32, kv_heads=8, head_dim=128)
QWEN3_32B = dict(hidden=5120, intermediate=25600, q_heads=64, kv_heads=8, head_dim=128)


def linear_shapes(model: dict) -> dict:
    """(K, N) of the four linear layers of one decoder block (nn.Linear: W is [N, K])."""
    H, I = model["hidden"], model["intermediate"]
    hq, hkv, d = model["q_heads"], model["kv_heads"], model["head_dim"]
    return {
        "qkv": (H, (hq + 2 * hkv) * d),
        "o": (hq * d, H),
        "gate_up": (H, 2 * I),
        "down": (I, H),
    }


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float values to bf16 (nearest even) and return the uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(seed: int, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    return to_bf16_bits(rng(seed).normal(mean, std, size=shape))


def heavy_tailed_bf16(seed: int, M: int, K: int, nu: float = 3.0, outlier_frac: float = 0.01,
                      outlier_gain: float = 20.0) -> np.ndarray:
    """Student-t(nu) activations with a fixed set of outlier channels.

    ceil(outlier_frac * K) column indices, drawn from the seed, are scaled by
    ``outlier_gain`` for every token (outlier channels shared by all tokens).
    """
    g = rng(seed)
    x = g.standard_t(nu, size=(M, K))
    n_out = int(np.ceil(outlier_frac * K))
    cols = g.choice(K, size=n_out, replace=False)
    x[:, cols] *= outlier_gain
    return to_bf16_bits(x)


def rms_weight_bf16(seed: int, H: int) -> np.ndarray:
    """RMSNorm weight ~ 1 + N(0, 0.1)."""
    return to_bf16_bits(1.0 + rng(seed).normal(0.0, 0.1, size=H))


def weight_bf16(seed: int, N: int, K: int, std: float = 0.02) -> np.ndarray:
    """Linear weight W [N, K] ~ N(0, std) (stand-in for a checkpoint)."""
    return to_bf16_bits(rng(seed).normal(0.0, std, size=(N, K)))


def random_e4m3_codes(seed: int, shape) -> np.ndarray:
    """Uniform random e4m3fn bytes, excluding the two NaN codes 0x7F / 0xFF."""
    g = rng(seed)
    c = g.integers(0, 254, size=shape, dtype=np.int64)
    c = np.where(c >= 0x7F, c + 1, c)            # skip 0x7F; 253 -> 254 (0xFE)
    return c.astype(np.uint8)


def random_scales(seed: int, shape, lo: float = 1e-3, hi: float = 1e-1) -> np.ndarray:
    """Positive fp32 scales, log-uniform in [lo, hi]."""
    g = rng(seed)
    return np.exp(g.uniform(np.log(lo), np.log(hi), size=shape)).astype(np.float32)


def random_pow2_scales(seed: int, shape, lo_exp: int = -12, hi_exp: int = -2) -> np.ndarray:
    g = rng(seed)
    return np.ldexp(1.0, g.integers(lo_exp, hi_exp + 1, size=shape)).astype(np.float32)


def random_e4m3_codes_u8(seed: int, shape) -> np.ndarray:
    """Uniform random positive finite e4m3fn bytes 0..125, drawn directly as
    uint8 (for large weight stand-ins where only the shape matters)."""
    return rng(seed).integers(0, 126, size=shape, dtype=np.uint8)
