"""Exact-arithmetic pins for the divisions in the oracle's quantizers.

The quantizers read the scale as ``s = max(fl32(amax / 7), 2**-126)`` and the code as
``clamp(round_half_even(fl32(w / s)))`` where ``fl32`` is one IEEE binary32 divide: the
exact quotient rounded once to the nearest fp32, ties to even (gemma ``uniform_quantize``
for the abs-max scale, ``round`` and ``clip``; LoopQ ``pack_weight`` for the quantizer
call; Keras ``quantize`` per-channel branch for the row-scale variant; Keras ``Dense``
merged-kernel helper, Step 3, for the LoRA re-quantize). Multiplying by a rounded
reciprocal instead (``amax * fl32(1/7)``, ``w * fl32(1/s)``) gives a different fp32 for
about half of all scales and moves codes that sit near a half-integer quotient.

Here every quotient is computed as an exact rational (``fractions.Fraction``) and rounded
to binary32 by integer arithmetic written in this file, so the expected codes and scales
depend on no floating-point divide. The rounding helper is itself pinned by hand-derived
binary32 patterns (ties, subnormals) before it is trusted. The inputs include groups built
so that a reciprocal multiply changes the scale or a code; planted reciprocal-multiply
mutants of the three quantizers each fail a pin below.
"""

import math
from fractions import Fraction

import numpy as np
import pytest

import oracle.w4_oracle as O
import workloads

FLT_MIN = Fraction(1, 2**126)


# ---------------------------------------------------------------------------
# binary32 rounding of an exact rational (the test's own, pinned below)
# ---------------------------------------------------------------------------

def fl32(r: Fraction) -> Fraction:
    """The binary32 value nearest to the rational ``r``, ties to an even significand.

    Normal numbers carry a 24-bit significand, so the quantum of a value in
    ``[2**e, 2**(e+1))`` is ``2**(e-23)``; below ``2**-126`` the quantum stays ``2**-149``
    (gradual underflow). The scaled value is rounded to an integer with Python's
    ``round`` on a Fraction, which sends ties to the even integer."""
    r = Fraction(r)
    if r == 0:
        return Fraction(0)
    a = abs(r)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while a >= Fraction(2) ** (e + 1):
        e += 1
    while a < Fraction(2) ** e:
        e -= 1
    quantum = Fraction(2) ** (max(e, -126) - 23)
    m = round(a / quantum)
    v = m * quantum
    if v > Fraction((2**24 - 1) * 2**104):
        raise OverflowError("beyond the largest binary32")
    return v if r > 0 else -v


def f32_bits(v: Fraction) -> int:
    """The binary32 bit pattern of a value that ``fl32`` returned (exact)."""
    return int(np.array([float(v)], np.float32).view(np.uint32)[0])


def _frac(x) -> Fraction:
    return Fraction(float(x))


# ---------------------------------------------------------------------------
# exact restatements of the three quantizers
# ---------------------------------------------------------------------------

def _rtn_block(w_vals, qmin, qmax):
    """One block of weights (a 32-column group or a whole row): the scale and codes."""
    amax = max(abs(_frac(w)) for w in w_vals)
    s = max(fl32(amax / 7), FLT_MIN)
    q = [min(max(round(fl32(_frac(w) / s)), qmin), qmax) for w in w_vals]
    return s, q


def rtn_exact(W):
    W = np.asarray(W, np.float32)
    N, K = W.shape
    G = math.ceil(K / 32)
    q = np.zeros((N, K), np.int64)
    s = np.zeros((N, G), np.float32)
    for n in range(N):
        for g in range(G):
            lo, hi = 32 * g, min(32 * g + 32, K)
            sg, qg = _rtn_block(W[n, lo:hi], -7, 7)
            s[n, g] = np.float32(float(sg))
            q[n, lo:hi] = qg
    return q, s


def rtn_channel_exact(W):
    W = np.asarray(W, np.float32)
    N, K = W.shape
    q = np.zeros((N, K), np.int64)
    s = np.zeros(N, np.float32)
    for n in range(N):
        sn, qn = _rtn_block(W[n], -8, 7)
        s[n] = np.float32(float(sn))
        q[n] = qn
    return q, s


def lora_merge_exact(q, s, b, a, c):
    """Merged weight with every fp32 step rounded as the oracle's reading states:
    ``w = fl32(q * s)``; ``t = fl32(t + fl32(b[n, j] * a[j, k]))`` for j in order;
    ``w' = fl32(w + fl32(c * t))``; then the exact group-32 quantizer."""
    N, K = q.shape
    r = b.shape[1]
    cf = _frac(np.float32(c))
    merged = np.zeros((N, K), np.float32)
    for n in range(N):
        for k in range(K):
            w = fl32(q[n, k] * _frac(s[n, k // 32]))
            t = Fraction(0)
            for j in range(r):
                t = fl32(t + fl32(_frac(b[n, j]) * _frac(a[j, k])))
            merged[n, k] = np.float32(float(fl32(w + fl32(cf * t))))
    return rtn_exact(merged)


# ---------------------------------------------------------------------------
# adversarial inputs: groups where a reciprocal multiply lands elsewhere
# ---------------------------------------------------------------------------

def _next_f32(x, steps):
    x = np.float32(x)
    toward = np.float32(np.inf) if steps > 0 else np.float32(-np.inf)
    for _ in range(abs(steps)):
        x = np.nextafter(x, toward)
    return x


def adversarial_rows(seed, n_rows, width=32):
    """Rows of ``width`` fp32 weights. Each row's largest magnitude ``A`` is one for which
    ``A * fl32(1/7)`` and ``A / 7`` round to different fp32 scales; most other entries sit
    within a few ulps of ``(k + 1/2) * s``, where the quotient's rounding decides the code.
    (NumPy only selects candidates here; the expected values come from :func:`rtn_exact`.)"""
    rng = np.random.default_rng(seed)
    rows = []
    inv7 = np.float32(1) / np.float32(7)
    while len(rows) < n_rows:
        A = np.float32(rng.uniform(0.004, 0.6))
        if A / np.float32(7) == A * inv7:
            continue
        s = A / np.float32(7)
        inv_s = np.float32(1) / s
        row = [A]
        for _ in range(4000):
            if len(row) >= (3 * width) // 4:
                break
            k = int(rng.integers(0, 7))
            w = _next_f32(np.float32((k + 0.5) * float(s)), int(rng.integers(-3, 4)))
            w = np.float32(-w if rng.random() < 0.5 else w)
            if np.rint(w / s) != np.rint(w * inv_s):
                row.append(w)
        while len(row) < width:
            row.append(np.float32(rng.uniform(-1, 1) * float(A)))
        row = np.array(row, np.float32)
        rng.shuffle(row)
        rows.append(row)
    return np.stack(rows)


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def pin_fl32_helper():
    """Hand-derived binary32 patterns: 1/3 = 0x3EAAAAAB (the 25th significand bit is 1 with
    a nonzero tail: round up); 1/7 = 0x3E124925; 2**24 + 1 is a tie and goes to the even
    2**24, 2**24 + 3 to 2**24 + 4; at the bottom of the range 2**-150 is a tie between 0
    and 2**-149 (goes to 0), 3 * 2**-150 between 2**-149 and 2**-148 (goes to 2**-148),
    5 * 2**-151 = 1.25 * 2**-149 goes to 2**-149; 2**-126 * (1 - 2**-25) rounds up to the
    smallest normal 0x00800000."""
    assert f32_bits(fl32(Fraction(1, 3))) == 0x3EAAAAAB
    assert f32_bits(fl32(Fraction(1, 7))) == 0x3E124925
    assert fl32(Fraction(2**24 + 1)) == 2**24
    assert fl32(Fraction(2**24 + 3)) == 2**24 + 4
    assert fl32(-Fraction(2**24 + 3)) == -(2**24 + 4)
    assert fl32(Fraction(1, 2**150)) == 0
    assert fl32(Fraction(3, 2**150)) == Fraction(1, 2**148)
    assert fl32(Fraction(5, 2**151)) == Fraction(1, 2**149)
    assert f32_bits(fl32(Fraction(1, 2**126) * (1 - Fraction(1, 2**25)))) == 0x00800000
    # IEEE 754 fixes the product and quotient of two binary32 numbers as exactly this
    # rounding: agree with the hardware's correctly rounded operations on random pairs
    rng = np.random.default_rng(11)
    a = (rng.standard_normal(300) * np.exp(rng.uniform(-30, 30, 300))).astype(np.float32)
    b = (rng.standard_normal(300) * np.exp(rng.uniform(-30, 30, 300))).astype(np.float32)
    for x, y in zip(a, b):
        assert np.float32(float(fl32(_frac(x) * _frac(y)))) == x * y
        assert np.float32(float(fl32(_frac(x) / _frac(y)))) == x / y


def pin_rtn_exact(o):
    """The group-32 quantizer against the exact-rational restatement, on random weights
    with outliers, a ragged last group, and the adversarial rows."""
    cases = [workloads.linear_case(31, 1, 6, 77, outliers=True)["W"],
             adversarial_rows(5, 24, 32).reshape(6, 128),
             adversarial_rows(6, 8, 32).reshape(4, 64)[:, :50]]
    for W in cases:
        q, s = o.quantize_rtn(W)
        qe, se = rtn_exact(W)
        assert np.array_equal(s, se), "scales differ from the exact quotient amax/7"
        assert np.array_equal(q.astype(np.int64), qe), "codes differ from rne(fl32(w/s))"


def pin_rtn_channel_exact(o):
    """The per-channel quantizer against its exact-rational restatement."""
    cases = [workloads.linear_case(32, 1, 5, 70, outliers=True)["W"],
             adversarial_rows(7, 12, 48)]
    for W in cases:
        q, s = o.quantize_rtn_channel(W)
        qe, se = rtn_channel_exact(W)
        assert np.array_equal(s, se), "row scales differ from the exact quotient amax/7"
        assert np.array_equal(q.astype(np.int64), qe), "codes differ from rne(fl32(w/s))"


def pin_lora_exact(o):
    """The LoRA merge (dequantize, rank-r update, re-quantize) against exact-rational
    steps, on an adapter large enough to move every group's scale."""
    rng = np.random.default_rng(33)
    N, K, r = 4, 70, 3
    W = workloads.linear_case(34, 1, N, K)["W"]
    q, s = O.quantize_rtn(W)
    b = (rng.standard_normal((N, r)) * 0.1).astype(np.float32)
    a = (rng.standard_normal((r, K)) * 0.1).astype(np.float32)
    c = 0.3
    q2, s2 = o.lora_merge(O.pack_nibbles(q), s, K, b, a, c)
    qe, se = lora_merge_exact(q.astype(np.int64), s, b, a, c)
    assert np.array_equal(s2, se), "merged scales differ from the exact steps"
    assert np.array_equal(q2.astype(np.int64), qe), "merged codes differ from the exact steps"


def test_fl32_helper():
    pin_fl32_helper()


def test_adversarial_rows_are_adversarial():
    """The constructed rows really separate the two readings: every row's scale differs
    under a reciprocal multiply, and so do many codes."""
    W = adversarial_rows(5, 24, 32)
    amax = np.max(np.abs(W), axis=1)
    assert np.all(amax / np.float32(7) != amax * (np.float32(1) / np.float32(7)))
    s = amax / np.float32(7)
    t_div = np.rint(W / s[:, None])
    t_mul = np.rint(W * (np.float32(1) / s)[:, None])
    assert np.count_nonzero(t_div != t_mul) >= 24 * 8


def test_rtn_exact_division():
    pin_rtn_exact(O)


def test_rtn_channel_exact_division():
    pin_rtn_channel_exact(O)


def test_lora_merge_exact_division():
    pin_lora_exact(O)


# ---------------------------------------------------------------------------
# planted mistakes: reciprocal multiplies instead of divides (on the CPU)
# ---------------------------------------------------------------------------

def _rtn_recip(W, scale_recip=True, code_recip=True):
    W = np.asarray(W, np.float32)
    N, K = W.shape
    G = math.ceil(K / 32)
    q = np.zeros((N, K), np.int8)
    sc = np.zeros((N, G), np.float32)
    inv7 = np.float32(1) / np.float32(7)
    for g in range(G):
        w = W[:, 32 * g: min(32 * g + 32, K)]
        amax = np.max(np.abs(w), axis=1)
        s = np.maximum(amax * inv7 if scale_recip else amax / np.float32(7), O.FLOOR)
        s = s.astype(np.float32)
        t = (w * (np.float32(1) / s)[:, None] if code_recip else w / s[:, None]).astype(np.float32)
        q[:, 32 * g: 32 * g + w.shape[1]] = np.clip(np.rint(t), -7, 7).astype(np.int8)
        sc[:, g] = s
    return q, sc


class _M:
    def __init__(self, **fns):
        self.quantize_rtn = fns.get("quantize_rtn", O.quantize_rtn)
        self.quantize_rtn_channel = fns.get("quantize_rtn_channel", O.quantize_rtn_channel)
        self.lora_merge = fns.get("lora_merge", O.lora_merge)


def _fails(pin, **fns):
    with pytest.raises(AssertionError):
        pin(_M(**fns))


def test_mutant_rtn_reciprocal_scale_and_code():
    _fails(pin_rtn_exact, quantize_rtn=_rtn_recip)


def test_mutant_rtn_reciprocal_code_only():
    """The scale divided correctly, only the code quotient taken as ``w * fl32(1/s)``."""
    _fails(pin_rtn_exact, quantize_rtn=lambda W: _rtn_recip(W, scale_recip=False))


def test_mutant_rtn_reciprocal_scale_only():
    _fails(pin_rtn_exact, quantize_rtn=lambda W: _rtn_recip(W, code_recip=False))


def test_mutant_channel_reciprocal():
    def q_recip(W):
        W = np.asarray(W, np.float32)
        amax = np.max(np.abs(W), axis=1)
        s = np.maximum(amax * (np.float32(1) / np.float32(7)), O.FLOOR).astype(np.float32)
        t = (W * (np.float32(1) / s)[:, None]).astype(np.float32)
        return np.clip(np.rint(t), -8, 7).astype(np.int8), s
    _fails(pin_rtn_channel_exact, quantize_rtn_channel=q_recip)


def test_mutant_channel_reciprocal_code_only():
    def q_recip(W):
        W = np.asarray(W, np.float32)
        s = np.maximum(np.max(np.abs(W), axis=1) / np.float32(7), O.FLOOR).astype(np.float32)
        t = (W * (np.float32(1) / s)[:, None]).astype(np.float32)
        return np.clip(np.rint(t), -8, 7).astype(np.int8), s
    _fails(pin_rtn_channel_exact, quantize_rtn_channel=q_recip)


def test_mutant_lora_requantize_reciprocal():
    def merge_recip(codes, scales, K, b, a, c):
        orig = O.quantize_rtn
        try:
            O.quantize_rtn = _rtn_recip
            return O.lora_merge(codes, scales, K, b, a, c)
        finally:
            O.quantize_rtn = orig
    _fails(pin_lora_exact, lora_merge=merge_recip)
