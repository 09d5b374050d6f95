"""Plain NumPy oracle for the GGUF Q4_0 block format and its linear y = x . dequant(W)^T + b.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU-baseline leg are
its only users; the library never calls it. Every function restates the definition below
with whole-array NumPy element operations and one float64 library matmul, nothing more.

Source: page "max/python/max/graph/quantization.py" (Modular MAX), class
``QuantizationEncoding`` (``Q4_0``: basic 4-bit quantization with 32 elements per block;
``is_gguf``) and its block-parameter table: a Q4_0 block encodes 32 elements in
``2 + 32 // 2`` = 18 bytes, the fields being the scale ``d`` and then the 4-bit codes ``q``.

Readings -- the page fixes only the element count, the byte count and the field order:

* ``d`` is an IEEE binary16 number stored little-endian in the block's first two bytes
  (a two-byte floating-point scale);
* the other 16 bytes hold 32 unsigned 4-bit codes c: element j of the block (0 <= j < 16)
  is the LOW nibble of code byte j and element j + 16 is its HIGH nibble (the GGUF layout);
* an element's value is ``d * (c - 8)``: the codes are centred on 8 (GGUF), computed in
  fp32, where the product is exact (11 significant bits times at most 4);
* a weight ``[N, K]`` (rows = output features, K a multiple of 32) is stored row-major as
  uint8 ``[N, K/32, 18]``: a row's blocks are consecutive, rows are consecutive.

Pins (tests): a hand-worked block, exact binary16 widening constants, a closed form (one-hot
x), and the reduction to the group-32 oracle: a block with ``d > 0`` is the packed group-32
format with scale ``d`` and signed codes ``c - 8`` (format v2 range [-8, 7]).
"""

from __future__ import annotations

import numpy as np

from . import w4_oracle as _w4

BLOCK = 32
"""Elements per block (page: ``BlockParameters(32, ...)`` for Q4_0)."""

BLOCK_BYTES = 18
"""Bytes per block (page: ``2 + 32 // 2``)."""

OFFSET = 8
"""Code offset: value = d * (c - 8) (reading, GGUF)."""


def unpack(blocks, K: int):
    """Split blocks into their fields.

    ``blocks`` uint8 ``[N, K/32, 18]``. Returns ``(d, c)``: ``d`` float32 ``[N, K/32]``
    (binary16 widened exactly) and ``c`` uint8 ``[N, K]``, the code of every element in
    column order (element j of block g is column 32g + j).
    """
    b = np.ascontiguousarray(blocks, dtype=np.uint8)
    if K % BLOCK != 0:
        raise ValueError("K must be a multiple of 32")
    N, G = b.shape[0], K // BLOCK
    if b.shape != (N, G, BLOCK_BYTES):
        raise ValueError(f"blocks must be [N, {G}, {BLOCK_BYTES}], got {b.shape}")
    d = np.ascontiguousarray(b[:, :, 0:2]).view("<f2")[:, :, 0].astype(np.float32)
    q = b[:, :, 2:]
    lo = q & np.uint8(0x0F)  # elements 0 .. 15 of the block
    hi = q >> np.uint8(4)    # elements 16 .. 31
    c = np.concatenate([lo, hi], axis=2).reshape(N, K)
    return d, c


def dequantize(blocks, K: int, out_dtype: str = "f32") -> np.ndarray:
    """``w[n, k] = fl32(d[n, k/32] * (c[n, k] - 8))``, then round to ``out_dtype``.

    ``out_dtype``: ``"f32"`` (float32), ``"f64"`` (exact widening), ``"bf16"`` (uint16 bit
    patterns, round-to-nearest-even) or ``"f16"`` (float16, round-to-nearest-even).
    """
    d, c = unpack(blocks, K)
    v = c.astype(np.float32) - np.float32(OFFSET)
    w = np.repeat(d, BLOCK, axis=1) * v
    if out_dtype == "f32":
        return w
    if out_dtype == "f64":
        return w.astype(np.float64)
    if out_dtype == "bf16":
        return _w4.f32_to_bf16_bits(w)
    if out_dtype == "f16":
        with np.errstate(over="ignore"):  # past 65504 rounds to infinity, as RNE does
            return w.astype(np.float16)
    raise ValueError(out_dtype)


def linear(x, blocks, K: int, bias=None):
    """Reference ``y[m, n] = sum_k x[m, k] * w[n, k] + b[n]`` in float64, with the dequantized
    fp32 weight of :func:`dequantize`, and the tolerance scale
    ``bound[m, n] = sum_k |x[m, k] * w[n, k]|``. ``x`` holds activation values as fp32
    (bf16 activations widen exactly). Returns ``(y_ref, bound)``, float64 ``[M, N]``."""
    w64 = dequantize(blocks, K, "f32").astype(np.float64)
    x64 = np.asarray(x, dtype=np.float32).astype(np.float64)
    y = x64 @ w64.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    bound = np.abs(x64) @ np.abs(w64).T
    return y, bound


def pack(d, c) -> np.ndarray:
    """Assemble blocks from scales and codes (the inverse of :func:`unpack`).

    ``d``: ``[N, G]`` values representable in binary16 (they are stored as float16);
    ``c``: ``[N, 32 G]`` integers in [0, 15]. Returns uint8 ``[N, G, 18]``.
    """
    c = np.asarray(c)
    if c.min(initial=0) < 0 or c.max(initial=0) > 15:
        raise ValueError("codes must lie in [0, 15]")
    N, K = c.shape
    G = K // BLOCK
    d16 = np.ascontiguousarray(np.asarray(d, dtype=np.float32).astype("<f2").reshape(N, G))
    dbytes = d16.view(np.uint8).reshape(N, G, 2)
    cb = c.astype(np.uint8).reshape(N, G, BLOCK)
    q = cb[:, :, :16] | (cb[:, :, 16:] << np.uint8(4))
    return np.concatenate([dbytes, q], axis=2)


def to_group32(blocks, K: int):
    """The blocks re-laid out as this library's packed group-32 format.

    A Q4_0 block is a group of 32 consecutive columns with one scale: element value
    ``d * (c - 8)`` is ``s * q`` with ``s = d`` (binary16 widened exactly to fp32) and the
    signed code ``q = c - 8`` in [-8, 7] (format v2). Returns ``(codes, scales)``: ``codes``
    uint8 ``[N, K/2]`` as :func:`w4_oracle.pack_nibbles` packs ``q`` (even column in the low
    nibble, two's complement), ``scales`` float32 ``[N, K/32]``. Every group-32 dequantization
    of the result equals :func:`dequantize` of the blocks (both products are exact)."""
    d, c = unpack(blocks, K)
    q = c.astype(np.int16) - OFFSET
    return _w4.pack_nibbles(q), d.astype(np.float32)


def validate(blocks, K: int) -> str:
    """"OK" when every block scale is finite, else "SCALE" (a reading: the page states no
    rule; a non-finite d turns every element of its block into NaN or infinity)."""
    d, _ = unpack(blocks, K)
    return "OK" if bool(np.all(np.isfinite(d))) else "SCALE"


def payload_bytes(N: int, K: int) -> int:
    """Bytes of a Q4_0 weight: 18 per block of 32 elements (4.5 bits per weight)."""
    return int(N) * (int(K) // BLOCK) * BLOCK_BYTES
