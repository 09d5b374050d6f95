"""Pins of the LoRA-merge oracle (Keras page, Dense's merged-kernel helper: dequantize,
add (alpha / rank) * A . B, re-quantize, pack): hand-worked merges with exact arithmetic
(tests/golden/lora_merge_worked_example.txt), the zero update reducing to re-quantizing the
dequantized weight (two pinned functions), a rank-one update equal to its closed form, and
planted mistakes that a pin must catch."""

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


PINS = [pin_lora_worked, pin_lora_zero_update, pin_lora_rank_one_closed_form]


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
