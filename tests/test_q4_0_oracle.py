"""Pins of the Q4_0 oracle (page "max/python/max/graph/quantization.py", QuantizationEncoding
.Q4_0 and its block parameters) against what the page and the mathematics fix: hand-worked
blocks (tests/golden/q4_0_worked_example.txt), binary16 constants, brute force over every
code byte, a closed form (one-hot activations) and the reduction to the already pinned
group-32 oracle."""

import numpy as np
import pytest

import oracle.q4_0 as Q
import oracle.w4_oracle as O
import workloads
from conftest import read_golden


def _hex(tokens):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def _nonzero(tokens, n):
    out = np.zeros(n)
    for tok in tokens:
        i, v = tok.split(":")
        out[int(i)] = float(v)
    return out


def pin_q4_0_worked(q):
    g = read_golden("q4_0_worked_example.txt")
    blk = _hex(g["A.bytes_hex"]).reshape(1, 1, 18)
    exp = np.array([float(v) for v in g["A.f32"]])
    assert np.array_equal(q.dequantize(blk, 32, "f32")[0].astype(np.float64), exp)
    x = _nonzero(g["A.x_nonzero"], 32).reshape(1, 32).astype(np.float32)
    y, bound = q.linear(x, blk, 32, np.array([float(g["A.bias"][0])], np.float32))
    assert y[0, 0] == float(g["A.y"][0])
    assert bound[0, 0] == abs(exp[0]) + 2 * abs(exp[16])
    blk = _hex(g["B.bytes_hex"]).reshape(1, 1, 18)
    w = q.dequantize(blk, 32, "f32")[0]
    assert np.all(w[:16] == float(g["B.f32_lo"][0])) and np.all(w[16:] == float(g["B.f32_hi"][0]))
    blk = _hex(g["C.bytes_hex"]).reshape(1, 1, 18)
    assert np.array_equal(q.dequantize(blk, 32, "f32")[0].astype(np.float64), _nonzero(g["C.f32_nonzero"], 32))
    blk = _hex(g["D.bytes_hex"]).reshape(1, 1, 18)
    assert np.array_equal(q.dequantize(blk, 32, "f32")[0].astype(np.float64), _nonzero(g["D.f32_nonzero"], 32))
    bf = O.bf16_bits_to_f32(q.dequantize(blk, 32, "bf16"))[0].astype(np.float64)
    assert np.array_equal(bf, _nonzero(g["D.bf16_nonzero"], 32))
    f16 = q.dequantize(blk, 32, "f16")[0].astype(np.float64)
    assert np.array_equal(f16, _nonzero(g["D.f16_nonzero"], 32))


def pin_q4_0_binary16(q):
    # binary16 bit patterns -> their values (IEEE 754: 5-bit exponent, bias 15, 10-bit fraction)
    cases = {0x0001: 2.0 ** -24, 0x03FF: 1023 * 2.0 ** -24, 0x0400: 2.0 ** -14, 0x3C00: 1.0,
             0x3555: 2.0 ** (13 - 15) * (1 + 0x155 / 1024), 0x7BFF: 65504.0, 0xC000: -2.0, 0x8000: -0.0}
    for bits, val in cases.items():
        blk = np.zeros((1, 1, 18), np.uint8)
        blk[0, 0, 0], blk[0, 0, 1] = bits & 0xFF, bits >> 8
        blk[0, 0, 2] = 0x09  # element 0: code 9 -> d * 1; element 16: code 0 -> d * -8
        d, c = q.unpack(blk, 32)
        assert d[0, 0] == val and np.signbit(d[0, 0]) == (bits >> 15 == 1), hex(bits)
        w = q.dequantize(blk, 32, "f32")[0]
        assert w[0] == val and w[16] == -8 * val


def pin_q4_0_code_bytes(q):
    # every byte value at every code position: low nibble -> element p, high -> element p + 16
    for p in range(16):
        blk = np.zeros((256, 1, 18), np.uint8)
        blk[:, 0, 1] = 0x3C  # d = 1.0
        blk[:, 0, 2:] = 0x88
        blk[:, 0, 2 + p] = np.arange(256, dtype=np.uint8)
        w = q.dequantize(blk, 32, "f32")
        b = np.arange(256)
        assert np.array_equal(w[:, p], (b & 15) - 8.0)
        assert np.array_equal(w[:, p + 16], (b >> 4) - 8.0)
        others = np.delete(w, [p, p + 16], axis=1)
        assert np.all(others == 0)


def pin_q4_0_one_hot(q):
    c = workloads.q4_0_case(3, 1, 24, 256)
    w = q.dequantize(c["blocks"], 256, "f32").astype(np.float64)
    for k in (0, 15, 16, 31, 32, 255):
        x = np.zeros((1, 256), np.float32)
        x[0, k] = 1.0
        y, _ = q.linear(x, c["blocks"], 256, c["bias"])
        assert np.array_equal(y[0], w[:, k] + c["bias"].astype(np.float64)), k


def pin_q4_0_group32_reduction(q):
    # d > 0: Q4_0 is the packed group-32 format with scale d and signed codes c - 8 (v2)
    rng = np.random.default_rng(11)
    N, K, M = 40, 320, 3
    d = np.abs(rng.standard_normal((N, K // 32)).astype(np.float32)).astype(np.float16) + np.float16(1e-3)
    c = rng.integers(0, 16, size=(N, K))
    blocks = q.pack(d.astype(np.float32), c)
    codes = O.pack_nibbles(c - 8)
    scales = d.astype(np.float32)
    assert np.array_equal(q.dequantize(blocks, K, "f32"), O.dequantize(codes, scales, K, "f32"))
    assert np.array_equal(q.dequantize(blocks, K, "bf16"), O.dequantize(codes, scales, K, "bf16"))
    x_bits, x = workloads.draw_x(rng, M, K)
    b = workloads.draw_bias(rng, N)
    y1, b1 = q.linear(x, blocks, K, b)
    y2, b2 = O.linear(x, codes, scales, K, b)
    assert np.array_equal(y1, y2) and np.array_equal(b1, b2)


def pin_q4_0_to_group32(q):
    # the re-laid-out weight dequantizes (group-32 oracle) to exactly the blocks' weight, for
    # scales of both signs, signed zero, a binary16 subnormal and the largest binary16 value,
    # and every code including c = 0 (q = -8)
    rng = np.random.default_rng(12)
    N, K = 9, 96
    d = (rng.standard_normal((N, K // 32)) * 0.01).astype(np.float32)
    d[0, 0], d[1, 1], d[2, 2], d[3, 0] = 0.0, -0.0, 2.0**-24, -65504.0
    c = rng.integers(0, 16, size=(N, K))
    c[0, :16] = np.arange(16)
    blocks = q.pack(d, c)
    codes, scales = q.to_group32(blocks, K)
    assert codes.dtype == np.uint8 and codes.shape == (N, K // 2)
    assert scales.dtype == np.float32 and scales.shape == (N, K // 32)
    assert np.array_equal(O.dequantize(codes, scales, K, "f32"), q.dequantize(blocks, K, "f32"))
    # by hand: columns 0 and 1 of row 0 hold codes 0 and 1, i.e. q = -8 and -7, nibbles 8 and 9
    assert codes[0, 0] == 0x98 and codes[0, 7] == 0x76  # columns 14, 15: q = 6, 7
    assert scales[2, 2] == np.float32(2.0**-24) and scales[3, 0] == np.float32(-65504.0)


def pin_q4_0_pack_roundtrip(q):
    blocks = workloads.q4_0_case(5, 1, 7, 96)["blocks"]
    d, c = q.unpack(blocks, 96)
    assert np.array_equal(q.pack(d, c), blocks)
    assert q.payload_bytes(7, 96) == blocks.size == 7 * 3 * 18


PINS = [pin_q4_0_worked, pin_q4_0_binary16, pin_q4_0_code_bytes, pin_q4_0_one_hot, pin_q4_0_group32_reduction,
        pin_q4_0_to_group32, pin_q4_0_pack_roundtrip]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_q4_0_pin(pin):
    pin(Q)


def test_q4_0_validate():
    blk = workloads.q4_0_case(1, 1, 3, 64)["blocks"].copy()
    assert Q.validate(blk, 64) == "OK"
    blk[1, 1, 0:2] = [0x00, 0x7C]  # +inf
    assert Q.validate(blk, 64) == "SCALE"


def test_q4_0_rejects_bad_shapes():
    with pytest.raises(ValueError):
        Q.unpack(np.zeros((2, 2, 18), np.uint8), 48)
    with pytest.raises(ValueError):
        Q.unpack(np.zeros((2, 3, 18), np.uint8), 64)


# ---------------------------------------------------------------------------
# planted mistakes (monkeypatched into the oracle, on the CPU): a pin must catch each
# ---------------------------------------------------------------------------

def _fails(pin):
    with pytest.raises(AssertionError):
        pin(Q)


def test_mutant_q4_0_nibble_halves_swapped(monkeypatch):
    orig = Q.unpack

    def unpack_swapped(blocks, K):
        d, c = orig(blocks, K)
        N = c.shape[0]
        cb = c.reshape(N, -1, 32)
        return d, np.concatenate([cb[:, :, 16:], cb[:, :, :16]], axis=2).reshape(N, K)
    monkeypatch.setattr(Q, "unpack", unpack_swapped)
    _fails(pin_q4_0_worked)
    _fails(pin_q4_0_code_bytes)


def test_mutant_q4_0_interleaved_nibbles(monkeypatch):
    # element 2j low / 2j + 1 high (the group-32 packing) instead of j / j + 16
    def unpack_interleaved(blocks, K):
        b = np.ascontiguousarray(blocks, dtype=np.uint8)
        N, G = b.shape[0], K // 32
        d = np.ascontiguousarray(b[:, :, 0:2]).view("<f2")[:, :, 0].astype(np.float32)
        q = b[:, :, 2:]
        c = np.stack([q & 15, q >> 4], axis=3).reshape(N, K)
        return d, c
    monkeypatch.setattr(Q, "unpack", unpack_interleaved)
    _fails(pin_q4_0_worked)


def test_mutant_q4_0_offset(monkeypatch):
    monkeypatch.setattr(Q, "OFFSET", 7)
    _fails(pin_q4_0_worked)
    _fails(pin_q4_0_code_bytes)


def test_mutant_q4_0_big_endian_scale(monkeypatch):
    orig = Q.unpack

    def unpack_be(blocks, K):
        _, c = orig(blocks, K)
        b = np.ascontiguousarray(blocks, dtype=np.uint8)
        d = np.ascontiguousarray(b[:, :, 0:2]).view(">f2")[:, :, 0].astype(np.float32)
        return d, c
    monkeypatch.setattr(Q, "unpack", unpack_be)
    _fails(pin_q4_0_worked)
    _fails(pin_q4_0_binary16)


def test_mutant_q4_0_scale_rounded_to_bf16(monkeypatch):
    # a plausible slip: the weight rounded to bf16 before the float64 contraction
    orig = Q.dequantize

    def deq_bf16(blocks, K, out_dtype="f32"):
        w = orig(blocks, K, out_dtype)
        if out_dtype == "f32":
            return O.bf16_bits_to_f32(O.f32_to_bf16_bits(w))
        return w
    monkeypatch.setattr(Q, "dequantize", deq_bf16)
    _fails(pin_q4_0_group32_reduction)


def test_mutant_q4_0_to_group32_bytes_copied(monkeypatch):
    # the block's code bytes copied as they are (element j / j + 16 per byte kept), offset applied
    def copied(blocks, K):
        b = np.ascontiguousarray(blocks, dtype=np.uint8)
        d = np.ascontiguousarray(b[:, :, 0:2]).view("<f2")[:, :, 0].astype(np.float32)
        return (b[:, :, 2:] ^ np.uint8(0x88)).reshape(b.shape[0], K // 2), d
    monkeypatch.setattr(Q, "to_group32", copied)
    _fails(pin_q4_0_to_group32)


def test_mutant_q4_0_to_group32_unsigned(monkeypatch):
    # codes c stored without the offset
    orig_unpack = Q.unpack

    def unsigned(blocks, K):
        d, c = orig_unpack(blocks, K)
        return O.pack_nibbles(c.astype(np.int16)), d
    monkeypatch.setattr(Q, "to_group32", unsigned)
    _fails(pin_q4_0_to_group32)
