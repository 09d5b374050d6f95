"""Pins of the input-gradient oracle ``linear_backward_x`` (Keras page, _int4_call grad_fn;
PaddleNLP page, QuantizationLinearFunc.backward): a hand-worked example
(tests/golden/backward_x_worked_example.txt), the adjointness identity with the pinned
forward linear (<y, dy> = <x, dx>, checked exactly in rational arithmetic on a small case),
a one-hot closed form, and planted mistakes that a pin must catch."""

from fractions import Fraction

import numpy as np
import pytest

import oracle.w4_oracle as O
import workloads
from conftest import read_golden


def _floats(tokens):
    return np.array([float(t) for t in tokens])


def pin_backward_worked(o):
    g = read_golden("backward_x_worked_example.txt")
    K = int(g["width"][0])
    codes = np.array([int(t, 16) for t in g["bytes_hex"]], np.uint8).reshape(2, -1)
    scales = _floats(g["scales"]).astype(np.float32).reshape(2, 1)
    dy = _floats(g["dy"]).astype(np.float32).reshape(1, 2)
    dx, bound = o.linear_backward_x(dy, codes, scales, K)
    assert np.array_equal(dx[0], _floats(g["dx"]))
    assert np.array_equal(bound[0], _floats(g["bound"]))


def pin_backward_adjoint_exact(o):
    # <y, dy> = <x, dx> for y = x . w^T (no bias): both sides are sums of the same products
    # x[m,k] w[n,k] dy[m,n]; in exact rational arithmetic they are equal, and the oracle's
    # float64 results, converted exactly, must match each within its rounding
    rng = np.random.default_rng(3)
    M, N, K = 2, 5, 70
    c = workloads.linear_case(9, M, N, K, bias=False)
    q, s = O.quantize_rtn(c["W"])
    codes = O.pack_nibbles(q)
    _, dy = workloads.draw_x(rng, M, N)
    y, _ = O.linear(c["x"], codes, s, K)
    dx, _ = o.linear_backward_x(dy, codes, s, K)
    w = O.dequantize(codes, s, K, "f32")
    lhs = sum(Fraction(float(dy[m, n])) * Fraction(float(c["x"][m, k])) * Fraction(float(w[n, k]))
              for m in range(M) for n in range(N) for k in range(K))
    got_y = sum(Fraction(float(y[m, n])) * Fraction(float(dy[m, n])) for m in range(M) for n in range(N))
    got_x = sum(Fraction(float(dx[m, k])) * Fraction(float(c["x"][m, k])) for m in range(M) for k in range(K))
    scale = sum(abs(Fraction(float(dy[m, n])) * Fraction(float(c["x"][m, k])) * Fraction(float(w[n, k])))
                for m in range(M) for n in range(N) for k in range(K))
    assert abs(got_y - lhs) <= scale * Fraction(1, 2 ** 40)
    assert abs(got_x - lhs) <= scale * Fraction(1, 2 ** 40)
    # and each dx element exactly: a sum of N exact products, rounded once per step in fp64
    for m in range(M):
        for k in range(0, K, 7):
            exact = sum(Fraction(float(dy[m, n])) * Fraction(float(w[n, k])) for n in range(N))
            mag = sum(abs(Fraction(float(dy[m, n])) * Fraction(float(w[n, k]))) for n in range(N))
            assert abs(Fraction(float(dx[m, k])) - exact) <= mag * Fraction(N, 2 ** 52)


def pin_backward_one_hot(o):
    c = workloads.linear_case(4, 1, 12, 96, bias=False)
    q, s = O.quantize_rtn(c["W"])
    codes = O.pack_nibbles(q)
    w = O.dequantize(codes, s, 96, "f32").astype(np.float64)
    for n in (0, 5, 11):
        dy = np.zeros((1, 12), np.float32)
        dy[0, n] = 1.0
        dx, bound = o.linear_backward_x(dy, codes, s, 96)
        assert np.array_equal(dx[0], w[n]) and np.array_equal(bound[0], np.abs(w[n]))


PINS = [pin_backward_worked, pin_backward_adjoint_exact, pin_backward_one_hot]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_backward_pin(pin):
    pin(O)


class _Mutant:
    """The oracle module with its backward replaced."""

    def __init__(self, fn):
        self.linear_backward_x = fn


def _fails(fn, pin):
    with pytest.raises(AssertionError):
        pin(_Mutant(fn))


def test_mutant_backward_wrong_row_index():
    # dy[m, n] paired with weight row N - 1 - n (a wrong index on the contracted axis)
    def bad(dy, codes, scales, K):
        w = O.dequantize(codes, scales, K, "f32").astype(np.float64)[::-1]
        dy64 = np.asarray(dy, np.float64)
        return dy64 @ w, np.abs(dy64) @ np.abs(w)
    _fails(bad, pin_backward_worked)
    _fails(bad, pin_backward_adjoint_exact)


def test_mutant_backward_scale_of_next_group():
    def bad(dy, codes, scales, K):
        s2 = np.roll(np.asarray(scales), 1, axis=1)
        w = O.dequantize(codes, s2, K, "f32").astype(np.float64)
        dy64 = np.asarray(dy, np.float64)
        return dy64 @ w, np.abs(dy64) @ np.abs(w)
    _fails(bad, pin_backward_adjoint_exact)


def test_mutant_backward_signed_bound():
    def bad(dy, codes, scales, K):
        dx, _ = O.linear_backward_x(dy, codes, scales, K)
        return dx, np.abs(dx)
    _fails(bad, pin_backward_worked)


def test_mutant_backward_weight_rounded_to_bf16():
    def bad(dy, codes, scales, K):
        w = O.bf16_bits_to_f32(O.dequantize(codes, scales, K, "bf16")).astype(np.float64)
        dy64 = np.asarray(dy, np.float64)
        return dy64 @ w, np.abs(dy64) @ np.abs(w)
    _fails(bad, pin_backward_adjoint_exact)
