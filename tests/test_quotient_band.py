"""The reciprocal quotient with an exact-division band, as the RTN quantizer and the LoRA
merge's re-quantize form their codes: with s = max(fl32(amax / 7), 2^-126), |w| <= amax and
y within one ulp of 1 / s, x = fl32(w * y) is rounded half to even (through the 2^23 bias)
unless |x - rne(x)| > 0.5 - 2^-18, where the IEEE quotient fl32(w / s) is rounded instead.
The claim is that this equals rne(fl32(w / s)) for every such w (the definition both kernels
are tested against). NumPy's float32 operations round to nearest even, so the argument is
checked here in the same arithmetic, for y = fl32(1 / s) and for both of its one-ulp
neighbours (the hardware reciprocal's error bound), on random groups and on values placed on
and next to every half-integer tie, the amax itself, zero, subnormal and the largest amax."""

import numpy as np

F32 = np.float32
BIAS = F32(12582912.0)  # 1.5 * 2^23
BAND = F32(0.5 - 2.0**-18)
TINY = np.finfo(np.float32).tiny


def scale_of(amax):
    return np.maximum((amax.astype(F32) / F32(7.0)).astype(F32), F32(TINY))


def band_codes(w, s, y):
    x = (w * y).astype(F32)
    xm = (x + BIAS).astype(F32)
    kf = (xm - BIAS).astype(F32)
    near = np.abs((x - kf).astype(F32)) > BAND
    exact = np.rint((w / s).astype(F32))
    return np.where(near, exact, kf), near


def reference_codes(w, s):
    return np.clip(np.rint((w / s).astype(F32)), -7, 7)


def check(w, amax):
    s = scale_of(amax)
    y0 = (F32(1.0) / s).astype(F32)
    for y in (y0, np.nextafter(y0, F32(np.inf)), np.nextafter(y0, F32(0.0))):
        got, _ = band_codes(w, s, y)
        ref = reference_codes(w, s)
        assert np.array_equal(got, ref), int(np.count_nonzero(got != ref))


def test_random_groups():
    rng = np.random.default_rng(20)
    n = 2_000_000
    amax = np.abs(rng.standard_normal(n) * 0.02).astype(F32) + F32(1e-30)
    w = (rng.uniform(-1.0, 1.0, n) * amax).astype(F32)
    w[::97] = amax[::97]
    w[1::97] = -amax[1::97]
    check(w, amax)


def test_ties_and_neighbours():
    # w placed on (k + 1/2) * s for every k in [-7, 6], and on the float32 values next to it
    rng = np.random.default_rng(21)
    n = 200_000
    amax = (np.abs(rng.standard_normal(n)) * F32(0.05) + F32(1e-3)).astype(F32)
    s = scale_of(amax)
    k = rng.integers(-7, 7, n).astype(F32) + F32(0.5)
    on = (k * s).astype(F32)
    for w in (on, np.nextafter(on, F32(np.inf)), np.nextafter(on, F32(-np.inf)),
              np.nextafter(np.nextafter(on, F32(np.inf)), F32(np.inf))):
        ok = np.abs(w) <= amax
        check(w[ok], amax[ok])


def test_band_is_taken_only_near_ties():
    rng = np.random.default_rng(22)
    n = 1_000_000
    amax = np.abs(rng.standard_normal(n)).astype(F32) + F32(1e-6)
    w = (rng.uniform(-1.0, 1.0, n) * amax).astype(F32)
    s = scale_of(amax)
    _, near = band_codes(w, s, (F32(1.0) / s).astype(F32))
    assert near.mean() < 1e-4  # about 2 * 2^-18 of uniform values
    k = np.rint((w / s).astype(F32))
    on = ((k + F32(0.5)) * s).astype(F32)
    ok = np.abs(on) <= amax
    _, near_on = band_codes(on[ok], s[ok], (F32(1.0) / s[ok]).astype(F32))
    assert near_on.mean() > 0.99  # values on a tie go to the exact quotient


def test_extreme_groups():
    big = np.array([np.finfo(np.float32).max] * 4, F32)
    w_big = np.array([big[0], -big[0], F32(big[0] / 3), F32(big[0] * 0.5)], F32)
    check(w_big, big)
    sub = np.array([F32(1e-45), F32(3e-42), F32(1e-39), F32(2e-38)], F32)  # subnormal amax: s = 2^-126
    check(np.array([F32(1e-45), -F32(3e-42), F32(5e-40), -F32(2e-38)], F32), sub)
    zero = np.zeros(4, F32)
    check(zero, zero)
    amax = np.full(16, F32(7.0))
    check(np.arange(-7.5, 8.5, 1.0, dtype=F32).clip(-7, 7), amax)  # s = 1: exact integers and ties


def test_mutant_band_removed_or_too_narrow(monkeypatch):
    # the fast path alone, or a band of 2^-24, rounds some ties and near-ties differently
    import pytest
    import test_quotient_band as T
    for band in (F32(1.0), F32(0.5 - 2.0**-24)):
        monkeypatch.setattr(T, "BAND", band)
        with pytest.raises(AssertionError):
            T.test_ties_and_neighbours()
