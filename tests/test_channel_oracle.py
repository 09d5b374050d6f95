"""Pins of the per-channel oracle (Keras page, quantize's per-channel branch, read as in
quantize_rtn_channel's docstring): a hand-worked example with exact quotients and ties
(tests/golden/channel_worked_example.txt), invariants (round trip within half a scale, a +-7
code in every row with a normal scale, sign symmetry, the code range), and the reduction to
the pinned group-32 oracle: a per-channel weight is a group-32 weight whose groups repeat
the row's scale."""

import numpy as np
import pytest

import oracle.w4_oracle as O
import workloads
from conftest import read_golden


def _f(tokens):
    return np.array([float(t) for t in tokens])


def pin_channel_worked(o):
    g = read_golden("channel_worked_example.txt")
    W = np.stack([_f(g["W0"]), _f(g["W1"]), _f(g["W2"])]).astype(np.float32)
    q, s = o.quantize_rtn_channel(W)
    assert np.array_equal(q, np.stack([_f(g["q0"]), _f(g["q1"]), _f(g["q2"])]).astype(np.int8))
    assert np.array_equal(s.astype(np.float64), _f(g["scales"]))
    codes = O.pack_nibbles(q)
    w = O.dequantize(codes, o.expand_channel_scales(s, 6), 6, "f32")
    assert np.array_equal(w[0].astype(np.float64), _f(g["w_hat0"]))


def pin_channel_invariants(o):
    c = workloads.linear_case(12, 1, 37, 333, outliers=True)
    W = c["W"]
    q, s = o.quantize_rtn_channel(W)
    assert q.min() >= -8 and q.max() <= 7 and s.shape == (37,) and np.all(s > 0) and np.all(np.isfinite(s))
    err = np.abs(W.astype(np.float64) - q.astype(np.float64) * s[:, None])
    assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 2.0 ** -20))
    assert np.all(np.abs(q).max(axis=1) == 7)
    q2, s2 = o.quantize_rtn_channel(-W)
    assert np.array_equal(s2, s) and np.array_equal(q2, -q)


def pin_channel_group_reduction(o):
    # a row whose every 32-column group has the same amax quantizes identically either way
    rng = np.random.default_rng(4)
    N, K = 6, 96
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    for g in range(K // 32):
        W[:, 32 * g] = 0.1  # the same amax in every group of every row
    q, s = o.quantize_rtn_channel(W)
    qg, sg = O.quantize_rtn(W)
    assert np.array_equal(q, qg) and np.array_equal(o.expand_channel_scales(s, K), sg)
    xb, x = workloads.draw_x(rng, 2, K)
    y1, b1 = O.linear(x, O.pack_nibbles(q), o.expand_channel_scales(s, K), K)
    y2, b2 = O.linear(x, O.pack_nibbles(qg), sg, K)
    assert np.array_equal(y1, y2) and np.array_equal(b1, b2)


PINS = [pin_channel_worked, pin_channel_invariants, pin_channel_group_reduction]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_channel_pin(pin):
    pin(O)


class _Mutant:
    def __init__(self, **fns):
        self.quantize_rtn_channel = fns.get("q", O.quantize_rtn_channel)
        self.expand_channel_scales = fns.get("e", O.expand_channel_scales)


def _fails(pin, **fns):
    with pytest.raises(AssertionError):
        pin(_Mutant(**fns))


def test_mutant_channel_scale_over_eight():
    def q8(W):
        W = np.asarray(W, np.float32)
        s = np.maximum(np.max(np.abs(W), axis=1) / np.float32(8), O.FLOOR).astype(np.float32)
        return np.clip(np.rint((W / s[:, None]).astype(np.float32)), -8, 7).astype(np.int8), s
    _fails(pin_channel_worked, q=q8)


def test_mutant_channel_rounds_half_away():
    def qa(W):
        W = np.asarray(W, np.float32)
        s = np.maximum(np.max(np.abs(W), axis=1) / np.float32(7), O.FLOOR).astype(np.float32)
        t = (W / s[:, None]).astype(np.float32)
        return np.clip(np.sign(t) * np.floor(np.abs(t) + 0.5), -8, 7).astype(np.int8), s
    _fails(pin_channel_worked, q=qa)


def test_mutant_channel_amax_over_columns():
    def qc(W):
        W = np.asarray(W, np.float32)
        s = np.maximum(np.max(np.abs(W), axis=0) / np.float32(7), O.FLOOR).astype(np.float32)
        s = np.resize(s, W.shape[0])
        return np.clip(np.rint((W / s[:, None]).astype(np.float32)), -8, 7).astype(np.int8), s
    _fails(pin_channel_worked, q=qc)
