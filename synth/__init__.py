"""Seeded synthetic inputs shared by the oracle-side tests and the CUDA-side tests.

This module draws random numbers and nothing else: it holds none of the
quantization, packing or matmul arithmetic. Both sides of every parity test
take their inputs from here, so the two implementations see the same bits.

Recipes (LLaMA-shaped layers stand in for real checkpoints; no model weights
or calibration datasets are used):

* weights: fp32 normal with a given std, optionally with a fraction of the
  entries replaced by std * Student-t(nu) (heavy tail), optionally with a
  seeded set of input channels (columns k) multiplied by a factor; rounded
  to fp16 at the end;
* activations: fp32 normal(0, 1), optionally with a seeded set of channels
  multiplied by a factor; rounded to fp16.

All generators use numpy's PCG64 via ``np.random.default_rng(seed)``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "rng",
    "outlier_channels",
    "weight",
    "activations",
    "LinearShape",
    "LLAMA2_7B_BLOCK",
    "LLAMA2_7B_AWQ_GROUPS",
    "config_small_linear",
    "config_llama7b_decode",
    "config_llama65b_decode",
    "config_smallm_sweep",
    "smallm_activations",
    "SMALLM_SWEEP",
    "config_awq_block",
]


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def outlier_channels(g: np.random.Generator, K: int, frac: float) -> np.ndarray:
    """ceil(frac*K) distinct channel indices chosen by a seeded permutation."""
    n = int(math.ceil(frac * K)) if frac > 0 else 0
    return np.sort(g.permutation(K)[:n])


def weight(g: np.random.Generator, N: int, K: int, std: float, *,
           channel_frac: float = 0.0, channel_mult: float = 1.0,
           heavy_frac: float = 0.0, heavy_nu: float = 3.0) -> np.ndarray:
    """fp16 weight [N][K] (nn.Linear layout: output rows, input columns)."""
    w = g.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    if heavy_frac > 0:
        cnt = int(round(heavy_frac * N * K))
        idx = g.choice(N * K, size=cnt, replace=False)
        w.reshape(-1)[idx] = (std * g.standard_t(heavy_nu, size=cnt)).astype(np.float32)
    if channel_frac > 0:
        ch = outlier_channels(g, K, channel_frac)
        w[:, ch] *= np.float32(channel_mult)
    return w.astype(np.float16)


def activations(g: np.random.Generator, M: int, K: int, *, std: float = 1.0,
                channel_frac: float = 0.0, channel_mult: float = 1.0) -> np.ndarray:
    """fp16 activations [M][K]."""
    x = g.standard_normal((M, K), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if channel_frac > 0:
        ch = outlier_channels(g, K, channel_frac)
        x[:, ch] *= np.float32(channel_mult)
    return x.astype(np.float16)


@dataclass(frozen=True)
class LinearShape:
    name: str
    K: int  # input channels
    N: int  # output channels


# LLaMA-2-7B decoder block: hidden 4096, MLP 11008.
LLAMA2_7B_BLOCK = (
    LinearShape("q_proj", 4096, 4096),
    LinearShape("k_proj", 4096, 4096),
    LinearShape("v_proj", 4096, 4096),
    LinearShape("o_proj", 4096, 4096),
    LinearShape("gate_proj", 4096, 11008),
    LinearShape("up_proj", 4096, 11008),
    LinearShape("down_proj", 11008, 4096),
)

# Linears that share one input activation, searched together by AWQ.
LLAMA2_7B_AWQ_GROUPS = (
    ("qkv", ("q_proj", "k_proj", "v_proj")),
    ("o", ("o_proj",)),
    ("gate_up", ("gate_proj", "up_proj")),
    ("down", ("down_proj",)),
)


@dataclass
class GemmCase:
    name: str
    X: np.ndarray          # [M][K] fp16
    W: np.ndarray          # [N][K] fp16
    bits: int = 4
    symmetric: bool = False
    extra: dict = field(default_factory=dict)


def config_small_linear(seed: int = 0) -> GemmCase:
    """Single linear K=256, N=128, M=1; 1% of input channels x10 in W."""
    g = rng(seed)
    W = weight(g, 128, 256, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = activations(g, 1, 256)
    return GemmCase("small_linear_K256_N128_M1", X, W)


def config_llama7b_decode(seed: int = 1, M: int = 1, shapes=LLAMA2_7B_BLOCK):
    """The 7 decode GEMVs of one LLaMA-2-7B block (W ~ N(0, 0.02), X ~ N(0, 1))."""
    g = rng(seed)
    out = []
    for s in shapes:
        W = weight(g, s.N, s.K, 0.02)
        X = activations(g, M, s.K)
        out.append(GemmCase(f"llama2_7b_{s.name}_K{s.K}_N{s.N}_M{M}", X, W))
    return out


def config_llama65b_decode(bits: int, seed: int = 2, M: int = 1, K: int = 8192, N: int = 8192) -> GemmCase:
    """[1,8192]x[8192,8192]: W ~ N(0,0.015) with 0.5% Student-t(3) entries; X with 1% channels x20."""
    g = rng(seed)
    W = weight(g, N, K, 0.015, heavy_frac=0.005, heavy_nu=3.0)
    X = activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    return GemmCase(f"llama65b_K{K}_N{N}_M{M}_b{bits}", X, W, bits=bits)


SMALLM_SWEEP = (1, 2, 4, 8, 16, 32, 64, 128)


def smallm_activations(M: int, seed: int = 4, K: int = 8192) -> np.ndarray:
    """The M fp16 rows ~ N(0, 1) of the small-M sweep (independent of the weight)."""
    return activations(rng(seed * 1000 + M), M, K)


def config_smallm_sweep(M: int, seed: int = 4, K: int = 8192, N: int = 28672) -> GemmCase:
    """K=8192, N=28672 weight (W ~ N(0, 0.01)) against M fp16 rows ~ N(0, 1)."""
    g = rng(seed)
    W = weight(g, N, K, 0.01)
    return GemmCase(f"smallm_K{K}_N{N}_M{M}", smallm_activations(M, seed, K), W)


def config_awq_block(seed: int = 5, T: int = 512, shapes=LLAMA2_7B_BLOCK,
                     groups=LLAMA2_7B_AWQ_GROUPS):
    """AWQ calibration of one LLaMA-2-7B block.

    Returns a list of (group_name, X_cal [T][K] fp16, [(linear_name, W [N][K] fp16), ...]).
    X_cal ~ N(0,1) with 1% of its channels x20; W ~ N(0, 0.02).
    """
    g = rng(seed)
    by_name = {s.name: s for s in shapes}
    out = []
    for gname, names in groups:
        K = by_name[names[0]].K
        X = activations(g, T, K, channel_frac=0.01, channel_mult=20.0)
        Ws = [(n, weight(g, by_name[n].N, K, 0.02)) for n in names]
        out.append((gname, X, Ws))
    return out
