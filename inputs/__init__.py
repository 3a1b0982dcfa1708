"""Seeded synthetic inputs for the AWQ W4A16 path (weights, activations, layer shapes).

This module is shared by the tests, the benchmark and the smoke check.  It holds
only random draws and shape tables: none of the quantizer's or the linear layer's
arithmetic lives here, so the CPU oracle and the CUDA library stay independent.

Recipe (stated once, used everywhere):
  * RNG: numpy ``Generator(PCG64(seed))``; values are drawn in float32, scaled,
    then rounded to float16 (round-to-nearest-even, numpy's cast).
  * W ~ N(0, sigma^2) with sigma = 0.02 (0.015 for the 70B-shaped prefill linears).
  * X ~ N(0, 1); exactly round(0.01*K) input channels, chosen without replacement
    from a separately seeded stream, are multiplied by 20 in every token row
    (the "~1% salient channels" that the AWQ pages describe as the ones
    activation statistics single out; see "AI-Research-SKILLs AWQ advanced usage
    guide", section 算法原理).
"""
from __future__ import annotations

import numpy as np

# Seed bases: weights, activations, outlier-channel set.  A workload adds its
# own offset and the linear's index within the workload.
SEED_W = 1000
SEED_X = 2000
SEED_OUTLIER = 3000

OUTLIER_FRACTION = 0.01
OUTLIER_MULT = 20.0

# One Mistral-7B decoder layer (hidden 4096, 8 KV heads of 128, MLP 14336):
# (name, K = in_features, N = out_features).
MISTRAL_7B_LAYER = (
    ("q_proj", 4096, 4096),
    ("k_proj", 4096, 1024),
    ("v_proj", 4096, 1024),
    ("o_proj", 4096, 4096),
    ("gate_proj", 4096, 14336),
    ("up_proj", 4096, 14336),
    ("down_proj", 14336, 4096),
)

# The same layer with q/k/v and gate/up concatenated row-wise (one weight matrix and
# one launch each), as the layer fusion of the AWQ inference path does:
# (name, K, N, [names of the concatenated linears]).
MISTRAL_7B_LAYER_FUSED = (
    ("qkv_proj", 4096, 6144, ("q_proj", "k_proj", "v_proj")),
    ("o_proj", 4096, 4096, ("o_proj",)),
    ("gate_up_proj", 4096, 28672, ("gate_proj", "up_proj")),
    ("down_proj", 14336, 4096, ("down_proj",)),
)

# Llama-70B-shaped prefill linears with q/k/v and gate/up fused:
# (name, K, N).
LLAMA_70B_FUSED = (
    ("qkv_proj", 8192, 10240),
    ("o_proj", 8192, 8192),
    ("gate_up_proj", 8192, 57344),
    ("down_proj", 28672, 8192),
)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def weights(n: int, k: int, sigma: float = 0.02, seed: int = SEED_W) -> np.ndarray:
    """fp16 weight matrix [n][k] (out x in), entries N(0, sigma^2)."""
    g = _rng(seed)
    w = g.standard_normal((n, k), dtype=np.float32) * np.float32(sigma)
    return w.astype(np.float16)


def outlier_channels(k: int, seed: int = SEED_OUTLIER) -> np.ndarray:
    """Sorted indices of the round(0.01*k) salient input channels."""
    count = int(round(OUTLIER_FRACTION * k))
    g = _rng(seed)
    return np.sort(g.choice(k, size=count, replace=False))


def activations(m: int, k: int, seed: int = SEED_X, outlier_seed: int = SEED_OUTLIER) -> np.ndarray:
    """fp16 activations [m][k]: N(0,1) with the outlier channels scaled x20."""
    g = _rng(seed)
    x = g.standard_normal((m, k), dtype=np.float32)
    idx = outlier_channels(k, outlier_seed)
    x[:, idx] *= np.float32(OUTLIER_MULT)
    return x.astype(np.float16)


def uniform_fp16(shape, lo: float, hi: float, seed: int) -> np.ndarray:
    """fp16 values uniform in [lo, hi) (used for edge-case tests)."""
    g = _rng(seed)
    return (g.random(shape, dtype=np.float32) * np.float32(hi - lo) + np.float32(lo)).astype(np.float16)


def random_codes(shape, seed: int) -> np.ndarray:
    """Uniform 4-bit codes 0..15 as uint8 (pack/unpack tests)."""
    return _rng(seed).integers(0, 16, size=shape, dtype=np.uint8)


def layer_inputs(shapes, m: int, sigma: float, seed_offset: int = 0):
    """Per-linear (name, W, X) for a list of (name, K, N) shapes.

    Linear i uses weight seed SEED_W + seed_offset + i and activation seed
    SEED_X + seed_offset + i; the outlier channel set depends only on K and the
    workload's offset, so every token row of one X shares it.
    """
    out = []
    for i, (name, k, n) in enumerate(shapes):
        w = weights(n, k, sigma, SEED_W + seed_offset + i)
        x = activations(m, k, SEED_X + seed_offset + i, SEED_OUTLIER + seed_offset)
        out.append((name, w, x))
    return out


def fused_layer_inputs(m: int, sigma: float, seed_offset: int = 0):
    """Per fused linear (name, W, X): the weights of the concatenated linears of
    MISTRAL_7B_LAYER (same seeds as layer_inputs) stacked row-wise, and the input of
    the first of them (the concatenated linears share their input)."""
    parts = {name: (w, x) for name, w, x in layer_inputs(MISTRAL_7B_LAYER, m, sigma, seed_offset)}
    out = []
    for name, k, n, members in MISTRAL_7B_LAYER_FUSED:
        w = np.concatenate([parts[mname][0] for mname in members], axis=0)
        assert w.shape == (n, k)
        out.append((name, w, parts[members[0]][1]))
    return out
