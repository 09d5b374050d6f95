"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and shapes them; it holds none of the
quantization, dequantization or matmul arithmetic, so both the CPU oracle and the
CUDA library can consume its outputs without sharing any method code.

Recipe (one NumPy PCG64 ``default_rng`` per case; draw order W, outlier mask, x,
bias, permutation):

* W   fp32 ``[N, K]`` ~ N(0, 0.02^2); with ``outliers`` 1% of entries (``random() <
  0.01``) are multiplied by 10.
* x   ``[M, K]`` ~ N(0, 1) drawn in fp32, rounded to bfloat16 (round-to-nearest-even
  by ``torch``); returned as bf16 bit patterns and as their exact fp32 values.
* b   fp32 ``[N]`` ~ N(0, 0.01^2).
* act-order ``g_idx`` int32 ``[K]``: a random permutation ``perm`` of the columns,
  ``g_idx[perm[j]] = j // group`` (each group owns ``group`` scattered columns).

The named workloads are the five configurations of the build: the small RTN
correctness case (seed 0), decode GEMV at M = 1, batched decode, prefill, and the
asymmetric act-order case; configuration ``c`` (1-based) other than the first
uses ``default_rng([0, c])``.
"""

from __future__ import annotations

import numpy as np
import torch

DECODE_SHAPES = ((4096, 4096), (14336, 4096), (4096, 14336))
"""(N, K) of the 4096-hidden decoder projections used for M = 1 decode."""
ODD_DEQUANT_SHAPE = (4096, 4095)
BATCHED_M = (8, 16, 32, 64)
BATCHED_SHAPE = (14336, 4096)
PREFILL_SHAPES = ((4096, 14336, 4096), (8192, 4096, 14336))
"""(M, N, K) prefill GEMMs."""
ASYM_SHAPE = (11008, 4096)
ASYM_GROUP = 128
ASYM_M = (1, 16, 2048)


def rng_for(config: int, salt: int | None = None) -> np.random.Generator:
    """Generator for configuration ``config`` (1-based); ``salt`` separates the
    several shapes inside one configuration."""
    if config == 1:
        return np.random.default_rng(0)
    key = [0, config] if salt is None else [0, config, salt]
    return np.random.default_rng(key)


def bf16_round(x_f32: np.ndarray):
    """fp32 samples -> (bf16 bit patterns uint16, their exact fp32 values)."""
    t = torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32)).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16).copy()
    vals = t.to(torch.float32).numpy().copy()
    return bits, vals


def draw_weight(rng: np.random.Generator, N: int, K: int, outliers: bool = False) -> np.ndarray:
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    if outliers:
        mask = rng.random((N, K)) < 0.01
        W = np.where(mask, W * np.float32(10), W).astype(np.float32)
    return W


def draw_x(rng: np.random.Generator, M: int, K: int):
    return bf16_round(rng.standard_normal((M, K), dtype=np.float32))


def draw_bias(rng: np.random.Generator, N: int) -> np.ndarray:
    return (rng.standard_normal(N, dtype=np.float32) * np.float32(0.01)).astype(np.float32)


def draw_act_order(rng: np.random.Generator, K: int, group: int):
    """Random act-order map: returns ``(g_idx int32 [K], perm int64 [K])``."""
    perm = rng.permutation(K)
    g_idx = np.empty(K, dtype=np.int32)
    g_idx[perm] = (np.arange(K) // group).astype(np.int32)
    return g_idx, perm


def linear_case(seed, M: int, N: int, K: int, outliers: bool = False, bias: bool = True):
    """A generic symmetric case: dict with W, x_bits, x, bias (or None)."""
    rng = np.random.default_rng(seed)
    W = draw_weight(rng, N, K, outliers)
    x_bits, x = draw_x(rng, M, K)
    b = draw_bias(rng, N) if bias else None
    return {"W": W, "x_bits": x_bits, "x": x, "bias": b, "M": M, "N": N, "K": K}


def config1():
    """RTN quantize + dequantize + linear, seed 0: W [256, 1000] with 1% x10
    outliers, x [4, 1000], fp32 bias."""
    rng = rng_for(1)
    W = draw_weight(rng, 256, 1000, outliers=True)
    x_bits, x = draw_x(rng, 4, 1000)
    b = draw_bias(rng, 256)
    return {"W": W, "x_bits": x_bits, "x": x, "bias": b, "M": 4, "N": 256, "K": 1000}


def decode_case(N: int, K: int, M: int = 1, config: int = 2, bias: bool = False):
    """Decode GEMV input: W ~ N(0, 0.02^2) [N, K] and x [M, K] (config 2 has no
    bias; config 3 draws one)."""
    rng = rng_for(config, salt=N * 100003 + K)
    W = draw_weight(rng, N, K)
    x_bits, x = draw_x(rng, M, K)
    b = draw_bias(rng, N) if bias else None
    return {"W": W, "x_bits": x_bits, "x": x, "bias": b, "M": M, "N": N, "K": K}


def asym_case(M: int, N: int = ASYM_SHAPE[0], K: int = ASYM_SHAPE[1], group: int = ASYM_GROUP,
              config: int = 5, seed=None):
    """Asymmetric act-order input: W [N, K], x [M, K], and the act-order map.
    The codes, scales and zero points are made from W by the oracle's min-max
    quantizer (test side) -- this module only draws the numbers."""
    rng = np.random.default_rng(seed) if seed is not None else rng_for(config, salt=M)
    W = draw_weight(rng, N, K)
    x_bits, x = draw_x(rng, M, K)
    b = draw_bias(rng, N)
    g_idx, perm = draw_act_order(rng, K, group)
    n_groups = (K + group - 1) // group
    return {"W": W, "x_bits": x_bits, "x": x, "bias": b, "g_idx": g_idx, "perm": perm,
            "n_groups": n_groups, "M": M, "N": N, "K": K, "group": group}


def asym_random_codes(M: int, N: int = ASYM_SHAPE[0], K: int = ASYM_SHAPE[1], group: int = ASYM_GROUP,
                      config: int = 5):
    """Asymmetric inputs drawn directly as random storage (for timing only): packed bytes of
    uniform unsigned nibbles (odd K: pad nibble zero), zero points uniform in [0, 15],
    scales uniform in [1e-3, 4e-3], plus x, bias and an act-order map as in ``asym_case``."""
    rng = rng_for(config, salt=1000 + M)
    P = (K + 1) // 2
    n_groups = (K + group - 1) // group
    codes = rng.integers(0, 256, size=(N, P), dtype=np.uint8)
    if K % 2:
        codes[:, -1] &= 0x0F
    zeros = rng.integers(0, 16, size=(N, n_groups)).astype(np.int8)
    scales = rng.uniform(1e-3, 4e-3, size=(N, n_groups)).astype(np.float32)
    x_bits, x = draw_x(rng, M, K)
    b = draw_bias(rng, N)
    g_idx, perm = draw_act_order(rng, K, group)
    return {"codes": codes, "zeros": zeros, "scales": scales, "x_bits": x_bits, "x": x, "bias": b,
            "g_idx": g_idx, "n_groups": n_groups, "M": M, "N": N, "K": K}


Q4_0_SHAPES = DECODE_SHAPES
"""(N, K) of the GGUF Q4_0 decode GEMVs (the same decoder projections)."""


def draw_q4_0_blocks(rng: np.random.Generator, N: int, K: int, d_sigma: float = 0.0056) -> np.ndarray:
    """Raw GGUF Q4_0 blocks, uint8 ``[N, K/32, 18]`` (K a multiple of 32): per block a
    binary16 scale ~ N(0, d_sigma^2) (both signs; the default is the size of a block scale
    of N(0, 0.02^2) weights), stored little-endian in bytes 0-1, then 16 code bytes drawn
    uniformly from [0, 255]. Only random draws and their storage layout, no arithmetic of
    the format."""
    G = K // 32
    d = (rng.standard_normal((N, G), dtype=np.float32) * np.float32(d_sigma)).astype("<f2")
    codes = rng.integers(0, 256, size=(N, G, 16), dtype=np.uint8)
    dbytes = np.ascontiguousarray(d).view(np.uint8).reshape(N, G, 2)
    return np.ascontiguousarray(np.concatenate([dbytes, codes], axis=2))


def q4_0_case(seed, M: int, N: int, K: int, bias: bool = True):
    """A Q4_0 linear case: dict with blocks, x_bits, x, bias (or None)."""
    rng = np.random.default_rng([1, int(seed)])
    blocks = draw_q4_0_blocks(rng, N, K)
    x_bits, x = draw_x(rng, M, K)
    b = draw_bias(rng, N) if bias else None
    return {"blocks": blocks, "x_bits": x_bits, "x": x, "bias": b, "M": M, "N": N, "K": K}
