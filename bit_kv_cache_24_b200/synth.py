"""Seeded synthetic inputs shaped like a 5B-class video DiT (3072 hidden, 24 heads x 128,
FFN 14336, 30 layers, 4680 tokens per autoregressive chunk).

This module only draws random BF16 tensors. It holds none of the NVFP4 arithmetic, so both the
CPU oracle (tests, bench cpu_baseline) and the CUDA path can be fed from it.

Streams: workload ``w`` uses seed ``w`` and every tensor of it draws from its own sub-stream
``j`` (numpy ``SeedSequence([seed, j])``), so a tensor's bytes do not depend on which other
tensors were generated before it.
"""
from __future__ import annotations

import math

import numpy as np
import torch

HIDDEN = 3072
HEADS = 24
HEAD_DIM = 128
FFN = 14336
LAYERS = 30
CHUNK_TOKENS = 4680          # 3 latent frames x 30 x 52 patches
KV_APPENDS = 12              # 12 x 4680 = 56160 cached tokens (global sink + shot sink + window)
TRAIN_TOKENS = 37440         # clean-history + noisy-target tokens of 4 chunks


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(stream)])))


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """float32/float64 numpy array -> torch bfloat16 (round to nearest even), CPU."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal(seed: int, stream: int, shape, std: float = 1.0) -> torch.Tensor:
    g = _rng(seed, stream)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return to_bf16(a)


def normal_with_outliers(seed: int, stream: int, shape, frac: float, factor: float) -> torch.Tensor:
    """N(0,1) where a Bernoulli(frac) subset of entries is multiplied by ``factor``."""
    g = _rng(seed, stream)
    a = g.standard_normal(size=shape, dtype=np.float32)
    mask = g.random(size=shape, dtype=np.float32) < np.float32(frac)
    a[mask] *= np.float32(factor)
    return to_bf16(a)


def channel_lognormal(seed: int, stream: int, rows: int, cols: int) -> torch.Tensor:
    """N(0,1) activations with a per-channel (column) scale drawn from LogNormal(0,1)."""
    g = _rng(seed, stream)
    scale = np.exp(g.standard_normal(size=(1, cols))).astype(np.float32)
    a = g.standard_normal(size=(rows, cols), dtype=np.float32)
    a *= scale
    return to_bf16(a)


def gelu_normal(seed: int, stream: int, rows: int, cols: int) -> torch.Tensor:
    """GELU (exact erf form, evaluated in float64) of N(0,1) samples: the FFN down-proj input."""
    g = _rng(seed, stream)
    z = torch.from_numpy(g.standard_normal(size=(rows, cols)))
    y = 0.5 * z * (1.0 + torch.erf(z / math.sqrt(2.0)))
    return y.to(torch.float32).to(torch.bfloat16)


def kv_outlier_channels(layer: int, seed: int = 4) -> np.ndarray:
    """Four outlier channels (out of heads*head_dim) for one layer, shared by K and V."""
    g = _rng(seed, 1000 + layer)
    return np.sort(g.choice(HEADS * HEAD_DIM, size=4, replace=False))


def kv_chunk(layer: int, append_idx: int, tokens: int = CHUNK_TOKENS, seed: int = 4):
    """K and V of one chunk for one layer: [tokens, 24, 128] ~N(0,1), 4 outlier channels x15."""
    ch = kv_outlier_channels(layer, seed)
    out = []
    for which in (0, 1):
        g = _rng(seed, 10_000 + (layer * 64 + append_idx) * 2 + which)
        a = g.standard_normal(size=(tokens, HEADS * HEAD_DIM), dtype=np.float32)
        a[:, ch] *= np.float32(15.0)
        out.append(to_bf16(a).view(tokens, HEADS, HEAD_DIM))
    return out[0], out[1]


# ---- the five workloads -------------------------------------------------------------------

def tiny(seed: int = 0):
    """Tiny W4A4 linear: A [128x256] N(0,1) with 1% entries x20, W [256x256] N(0,0.02)."""
    return {
        "A": normal_with_outliers(seed, 0, (128, 256), 0.01, 20.0),
        "W": normal(seed, 1, (256, 256), 0.02),
    }


def qkv(seed: int = 1, tokens: int = CHUNK_TOKENS):
    """QKV projection of one chunk: A [4680x3072] (per-channel LogNormal scale), W [9216x3072]
    N(0,0.02), bias [9216] N(0,0.02)."""
    return {
        "A": channel_lognormal(seed, 0, tokens, HIDDEN),
        "W": normal(seed, 1, (3 * HIDDEN, HIDDEN), 0.02),
        "bias": normal(seed, 2, (3 * HIDDEN,), 0.02),
    }


def ffn(seed: int = 2, tokens: int = CHUNK_TOKENS):
    """FFN of one chunk: up-proj [4680x3072]x[14336x3072]^T, down-proj GELU input
    [4680x14336]x[3072x14336]^T with a residual R [4680x3072] N(0,1)."""
    return {
        "A_up": channel_lognormal(seed, 0, tokens, HIDDEN),
        "W_up": normal(seed, 1, (FFN, HIDDEN), 0.02),
        "A_down": gelu_normal(seed, 2, tokens, FFN),
        "W_down": normal(seed, 3, (HIDDEN, FFN), 0.02),
        "R": normal(seed, 4, (tokens, HIDDEN)),
    }


def train(seed: int = 3, tokens: int = TRAIN_TOKENS):
    """Training-shape GEMM operands: X [37440x3072] (per-channel LogNormal), dY N(0,1),
    W [3072x3072] N(0,0.02)."""
    return {
        "X": channel_lognormal(seed, 0, tokens, HIDDEN),
        "dY": normal(seed, 1, (tokens, HIDDEN)),
        "W": normal(seed, 2, (HIDDEN, HIDDEN), 0.02),
    }


def ragged(seed: int, rows: int, cols: int, kind: str = "normal") -> torch.Tensor:
    """Small test tensors of arbitrary shape; ``kind`` picks the value distribution."""
    if kind == "normal":
        return normal(seed, 0, (rows, cols))
    if kind == "outliers":
        return normal_with_outliers(seed, 0, (rows, cols), 0.01, 20.0)
    if kind == "lognormal":
        return channel_lognormal(seed, 0, rows, cols)
    if kind == "wide":
        # magnitudes spread over many binades, exercising E4M3 subnormal and saturated scales
        g = _rng(seed, 0)
        a = g.standard_normal(size=(rows, cols)) * np.exp2(g.integers(-40, 40, size=(rows, 1)))
        return to_bf16(a.astype(np.float32))
    raise ValueError(kind)
