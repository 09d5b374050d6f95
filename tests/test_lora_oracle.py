"""Pins of the LoRA-merge oracle (Keras page, Dense's merged-kernel helper: dequantize,
add (alpha / rank) * A . B, re-quantize, pack): hand-worked merges with exact arithmetic
(tests/golden/lora_merge_worked_example.txt), the zero update reducing to re-quantizing the
dequantized weight (two pinned functions), a rank-one update equal to its closed form,
merged values on and 2^-22 beside half-integers re-quantizing half to even, and planted
mistakes that a pin must catch."""

import numpy as np
import pytest

import oracle.w4_oracle as O
import workloads
from conftest import read_golden


def _f(tokens):
    return np.array([float(t) for t in tokens])


def pin_lora_worked(o):
    g = read_golden("lora_merge_worked_example.txt")
    codes = np.array([int(t, 16) for t in g["codes_hex"]], np.uint8).reshape(1, 2)
    s = _f(g["scales"]).astype(np.float32).reshape(1, 1)
    for case, rows in (("c1", ["a0"]), ("c2", ["a0", "a1"])):
        b = _f(g[case + ".b"]).astype(np.float32).reshape(1, -1)
        a = np.stack([_f(g[f"{case}.{r}"]) for r in rows]).astype(np.float32)
        q, s2 = o.lora_merge(codes, s, 4, b, a, float(g[case + ".c"][0]))
        assert np.array_equal(q[0].astype(np.float64), _f(g[case + ".q"])), case
        assert np.array_equal(s2.astype(np.float64).ravel(), _f(g[case + ".s"])), case


def pin_lora_zero_update(o):
    c = workloads.linear_case(6, 1, 20, 200)
    q, s = O.quantize_rtn(c["W"])
    codes = O.pack_nibbles(q)
    b = np.zeros((20, 4), np.float32)
    a = np.random.default_rng(1).standard_normal((4, 200)).astype(np.float32)
    q2, s2 = o.lora_merge(codes, s, 200, b, a, 2.0)
    q3, s3 = O.quantize_rtn(O.dequantize(codes, s, 200, "f32"))
    assert np.array_equal(q2, q3) and np.array_equal(s2, s3)


def pin_lora_rank_one_closed_form(o):
    # r = 1, c = 1: the merged weight is w + b a exactly when every product is exact
    # (powers of two): the re-quantized codes must be those of that weight
    N, K = 3, 64
    rng = np.random.default_rng(2)
    q0 = rng.integers(-7, 8, size=(N, K))
    s = np.full((N, 2), 0.25, np.float32)
    codes = O.pack_nibbles(q0)
    b = np.array([[1.0], [-0.5], [2.0]], np.float32)
    a = (rng.integers(-4, 5, size=(1, K)) * 0.125).astype(np.float32)
    q, s2 = o.lora_merge(codes, s, K, b, a, 1.0)
    exact = q0 * 0.25 + b @ a
    q3, s3 = O.quantize_rtn(exact.astype(np.float32))
    assert np.array_equal(q, q3) and np.array_equal(s2, s3)


# offsets of the merged value from its code q: exact half-integer ties and values 2^-22 to
# either side of one (exact in fp32 while |q + d| < 4), and 0
TIE_OFFSETS = (0.5, -0.5, 0.5 + 2.0**-22, 0.5 - 2.0**-22, -0.5 + 2.0**-22, -0.5 - 2.0**-22, 1.5, -1.5, 0.0)


def lora_tie_case(row_scales):
    """A rank-one merge (c = 1) whose merged values sit on or 2^-22 beside half-integers of
    the row's scale: K = 64 (two groups); column 0 of each group keeps code 7 and offset 0, so
    the group's amax is 7 s and its new scale s again; the other columns take codes in
    -3 .. 2 and an offset d from TIE_OFFSETS through b[n] = s[n], a[0, k] = d. Returns
    (codes, scales, b, a, q, d) with q and d the [N, 64] codes and offsets."""
    N, K = len(row_scales), 64
    q = np.zeros((N, K), np.int64)
    d = np.zeros((N, K))
    qs = (-3, -2, -1, 0, 1, 2)
    for n in range(N):
        for k in range(K):
            if k % 32 == 0:
                q[n, k] = 7
            else:
                q[n, k] = qs[(5 * k + n) % len(qs)]
                d[n, k] = TIE_OFFSETS[k % len(TIE_OFFSETS)]
    # one offset per column: rows share a (rank one), so every row takes column k's offset
    d[:] = d[0]
    s = np.repeat(np.asarray(row_scales, np.float32).reshape(N, 1), 2, axis=1)
    b = np.asarray(row_scales, np.float32).reshape(N, 1)
    a = d[0:1].astype(np.float32)
    return O.pack_nibbles(q), s, b, a, q, d


def pin_lora_half_even_ties(o):
    # unit scales: every step is exact, so the new codes are round-half-even(q + d) and the
    # scales stay 1
    codes, s, b, a, q, d = lora_tie_case([1.0, 1.0, 1.0])
    q2, s2 = o.lora_merge(codes, s, 64, b, a, 1.0)
    expect = np.vectorize(lambda v: round(v))(q + d)  # Python's round() is half to even
    assert np.array_equal(q2.astype(np.int64), expect)
    assert np.array_equal(s2, np.ones_like(s2))


PINS = [pin_lora_worked, pin_lora_zero_update, pin_lora_rank_one_closed_form, pin_lora_half_even_ties]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_lora_pin(pin):
    pin(O)


class _Mutant:
    def __init__(self, fn):
        self.lora_merge = fn


def _fails(fn, pin):
    with pytest.raises(AssertionError):
        pin(_Mutant(fn))


def _merge(codes, scales, K, b, a, c, sign=1.0, use_c=True, transpose=False):
    w = O.dequantize(codes, scales, K, "f32")
    b = np.asarray(b, np.float32)
    a = np.asarray(a, np.float32)
    t = (b @ a).astype(np.float32) if not transpose else (b @ a[::-1]).astype(np.float32)
    d = (np.float32(c) * t if use_c else t).astype(np.float32)
    return O.quantize_rtn((w + np.float32(sign) * d).astype(np.float32))


def test_mutant_lora_sign_flipped():
    _fails(lambda *args: _merge(*args, sign=-1.0), pin_lora_worked)


def test_mutant_lora_alpha_ignored():
    _fails(lambda *args: _merge(*args, use_c=False), pin_lora_worked)


def test_mutant_lora_rank_rows_swapped():
    _fails(lambda *args: _merge(*args, transpose=True), pin_lora_worked)


def _merge_half_away(codes, scales, K, b, a, c):
    w = O.dequantize(codes, scales, K, "f32")
    t = (np.asarray(b, np.float32) @ np.asarray(a, np.float32)).astype(np.float32)
    m = (w + (np.float32(c) * t).astype(np.float32)).astype(np.float32)
    g = m.reshape(m.shape[0], -1, 32)
    s2 = np.maximum((np.abs(g).max(axis=2) / np.float32(7)).astype(np.float32), np.finfo(np.float32).tiny)
    x = (g / s2[:, :, None]).astype(np.float32)
    qq = np.clip(np.sign(x) * np.floor(np.abs(x) + 0.5), -7, 7).astype(np.int8)
    return qq.reshape(m.shape), s2.astype(np.float32)


def test_mutant_lora_ties_away_from_zero():
    codes, s, b, a = lora_tie_case([1.0])[:4]
    assert np.array_equal(_merge_half_away(codes, s, 64, b, a, 1.0)[1], np.ones((1, 2), np.float32))
    _fails(_merge_half_away, pin_lora_half_even_ties)
