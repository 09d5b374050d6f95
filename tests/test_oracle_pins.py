"""Pins for the CPU oracle: it is checked against what the source pages and the
mathematics fix -- hand-worked examples (tests/golden, each citing its page),
closed forms, invariants, brute force over all byte values, exact rational
arithmetic on tiny inputs, and special cases that reduce to a library routine.

The ``pin_*`` functions take the oracle module so that test_oracle_mutations.py
can run them against planted mistakes and confirm each mistake is caught.
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.w4_oracle as O
import workloads
from conftest import read_golden


def _hex(tokens):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def _floats(tokens):
    return np.array([float(t) for t in tokens], dtype=np.float64)


def _ints(tokens):
    return np.array([int(t) for t in tokens], dtype=np.int64)


# ---------------------------------------------------------------------------
# pins (each raises AssertionError on a mismatch)
# ---------------------------------------------------------------------------

def pin_bf16_rne(o):
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),  # subnormals
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.01171875, -1.00390625,
                  65504.0, 3.3895314e38, np.inf, -np.inf, 1e-45, -1e-45], np.float32),
    ])
    # every fp32 with a low half of exactly 0x8000 is a bf16 tie
    ties = (rng.integers(0, 2**16, 4000, dtype=np.uint32) << 16 | 0x8000).astype(np.uint32)
    ties = ties.view(np.float32)
    ties = ties[np.isfinite(ties)]
    vals = np.concatenate([vals, ties])
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = o.f32_to_bf16_bits(vals)
    assert np.array_equal(got, ref), "bf16 RNE differs from torch"
    back = o.bf16_bits_to_f32(got)
    assert np.array_equal(back, torch.from_numpy(got.view(np.int16)).view(torch.bfloat16).float().numpy())


def pin_pack_worked(o):
    g = read_golden("pack_worked_example.txt")
    K = int(g["width"][0])
    vals = _ints(g["values"]).reshape(1, K)
    codes = o.pack_nibbles(vals)
    assert codes.shape == (1, math.ceil(K / 2))
    assert np.array_equal(codes[0], _hex(g["bytes_hex"])), codes
    assert np.array_equal(o.unpack_signed(codes, K)[0], vals[0])
    rb = _hex(g["reserved_byte_hex"]).reshape(1, 1)
    assert np.array_equal(o.unpack_signed(rb, 2)[0], _ints(g["reserved_values"]))
    assert o.validate(rb, np.ones((1, 1), np.float32), 2, 2) == "OK"
    assert o.validate(rb, np.ones((1, 1), np.float32), 2, 1) == "RESERVED_CODE"


def pin_unpack_brute_force(o):
    """All 256 byte values: unpack then pack is the identity; exactly 31 bytes
    carry the nibble 8 (16 + 16 - 1) and only those fail format v1; the 240
    bytes with a nonzero high nibble fail as the last byte of an odd width."""
    allb = np.arange(256, dtype=np.uint8).reshape(256, 1)
    vals = o.unpack_signed(allb, 2)
    assert vals.min() == -8 and vals.max() == 7
    for b in range(256):
        lo, hi = b & 15, b >> 4
        assert vals[b, 0] == (lo - 16 if lo >= 8 else lo)
        assert vals[b, 1] == (hi - 16 if hi >= 8 else hi)
    assert np.array_equal(o.pack_nibbles(vals)[:, 0], allb[:, 0])
    one = np.ones((1, 1), np.float32)
    v1_rejected = [b for b in range(256)
                   if o.validate(np.array([[b]], np.uint8), one, 2, 1) == "RESERVED_CODE"]
    assert len(v1_rejected) == 31
    assert all((b & 15) == 8 or (b >> 4) == 8 for b in v1_rejected)
    odd_rejected = [b for b in range(256)
                    if o.validate(np.array([[b]], np.uint8), one, 1, 2) == "HIGH_NIBBLE"]
    assert len(odd_rejected) == 240 and all(b >> 4 for b in odd_rejected)
    # odd width truncates: the unused high nibble never shows up
    assert o.unpack_signed(np.array([[0x97]], np.uint8), 1).shape == (1, 1)


def pin_rtn_worked(o):
    g = read_golden("rtn_worked_example.txt")
    for case in "ABCD":
        K = int(g[case + ".width"][0])
        w = _floats(g[case + ".w"]).astype(np.float32).reshape(1, K)
        q, s = o.quantize_rtn(w)
        assert np.array_equal(q[0].astype(np.int64), _ints(g[case + ".q"])), (case, q)
        assert np.array_equal(s[0], _floats(g[case + ".scales"]).astype(np.float32)), (case, s)


def pin_rtn_invariants(o, W):
    W = np.asarray(W, np.float32)
    q, s = o.quantize_rtn(W)
    N, K = W.shape
    G = math.ceil(K / 32)
    assert q.shape == (N, K) and s.shape == (N, G) and s.dtype == np.float32
    assert q.min() >= -7 and q.max() <= 7
    assert np.isfinite(s).all() and (s > 0).all()
    s_full = np.repeat(s.astype(np.float64), 32, axis=1)[:, :K]
    err = np.abs(W.astype(np.float64) - q.astype(np.float64) * s_full)
    assert (err <= s_full * (0.5 + 2.0**-20)).all(), "round-trip error above scale/2"
    # each group whose amax/7 is normal reaches a code of magnitude 7
    for g in range(G):
        blk = np.abs(W[:, 32 * g: 32 * g + 32])
        big = blk.max(axis=1) >= 7 * np.finfo(np.float32).tiny
        assert (np.abs(q[big, 32 * g: 32 * g + 32]).max(axis=1) == 7).all()
    # w -> -w maps q -> -q with the same scales (RNE is symmetric)
    q2, s2 = o.quantize_rtn(-W)
    assert np.array_equal(s2, s) and np.array_equal(q2, -q)


def pin_dequant_worked(o):
    g = read_golden("dequant_worked_example.txt")
    for case in "PR":
        K = int(g[case + ".width"][0])
        codes = _hex(g[case + ".bytes_hex"]).reshape(1, -1)
        s = _floats(g[case + ".scales"]).astype(np.float32).reshape(1, -1)
        exp = _floats(g[case + ".f32"])
        assert np.array_equal(o.dequantize(codes, s, K, "f32")[0].astype(np.float64), exp), case
        assert np.array_equal(o.dequantize(codes, s, K, "f64")[0], exp), case
        assert np.array_equal(o.dequantize(codes, s, K, "f16")[0].astype(np.float64), exp), case
    K = int(g["T.width"][0])
    codes = _hex(g["T.bytes_hex"]).reshape(1, -1)
    assert codes.shape[1] == math.ceil(K / 2)
    s = _floats(g["T.scales"]).astype(np.float32).reshape(1, -1)
    f32 = o.dequantize(codes, s, K, "f32")[0]
    bf = o.bf16_bits_to_f32(o.dequantize(codes, s, K, "bf16"))[0]
    exp_f = np.zeros(K)
    exp_b = np.zeros(K)
    for tok in g["T.f32_nonzero"]:
        i, v = tok.split(":")
        exp_f[int(i)] = float(v)
    for tok in g["T.bf16_nonzero"]:
        i, v = tok.split(":")
        exp_b[int(i)] = float(v)
    assert np.array_equal(f32.astype(np.float64), exp_f)
    assert np.array_equal(bf.astype(np.float64), exp_b)


def pin_dequant_closed_form(o):
    """Power-of-two scales make every product exact in every output dtype, so the
    dequantized value must be exactly code * scale, for any width (ragged too)."""
    rng = np.random.default_rng(3)
    for K in (1, 5, 32, 33, 63, 64, 100):
        N = 7
        vals = rng.integers(-8, 8, size=(N, K))
        codes = o.pack_nibbles(vals)
        G = math.ceil(K / 32)
        s = (2.0 ** rng.integers(-20, 10, size=(N, G))).astype(np.float32)
        exp = vals * np.repeat(s.astype(np.float64), 32, axis=1)[:, :K]
        for dt in ("f32", "f64", "f16"):
            got = o.dequantize(codes, s, K, dt).astype(np.float64)
            if dt == "f16":
                ok = np.abs(exp) <= 65504
                ok &= (np.abs(exp) >= 2.0**-14) | (exp == 0)
                assert np.array_equal(got[ok], exp[ok])
            else:
                assert np.array_equal(got, exp)
        got = o.bf16_bits_to_f32(o.dequantize(codes, s, K, "bf16")).astype(np.float64)
        assert np.array_equal(got, exp)


def pin_linear_worked(o):
    g = read_golden("linear_worked_example.txt")
    K = int(g["width"][0])
    q = np.stack([_ints(g["q0"]), _ints(g["q1"])])
    codes = o.pack_nibbles(q)
    s = _floats(g["scales"]).astype(np.float32).reshape(2, 1)
    x = _floats(g["x"]).astype(np.float32).reshape(1, K)
    b = _floats(g["bias"]).astype(np.float32)
    y, bound = o.linear(x, codes, s, K, b)
    assert np.array_equal(y[0], _floats(g["y"])), y
    assert np.array_equal(bound[0], _floats(g["bound"])), bound


def pin_check_linear(o):
    """The acceptance rule ``|y - y_ref| <= 4e-3 * bound + 1e-6`` (the linear tolerance),
    element by element, with values chosen so that every allowance is an exact double:
    ``4e-3 * 1000`` rounds to exactly 4, so the allowance there is ``4 + 1e-6``; with a
    zero bound it is ``1e-6``. An error equal to the allowance passes, the next double
    above it fails, an error below ``y_ref`` counts as much as one above, and one bad
    element (or a NaN) among many fails the whole output."""
    y_ref = np.zeros((4, 2500))
    bound = np.full((4, 2500), 1000.0)
    bound[1] = 0.0
    allow = np.where(bound > 0, 4.000001, 1e-6)
    assert np.array_equal(4e-3 * bound + 1e-6, allow)
    ok, worst = o.check_linear(y_ref + allow, y_ref, bound)
    assert ok and worst == 1.0, (ok, worst)
    ok, _ = o.check_linear(y_ref - allow, y_ref, bound)
    assert ok
    for m, n, sign in [(0, 7, 1.0), (1, 2499, -1.0), (3, 1234, 1.0)]:
        y = y_ref + 0.5 * allow
        y[m, n] = sign * np.nextafter(allow[m, n], np.inf)
        ok, worst = o.check_linear(y, y_ref, bound)
        assert not ok and worst > 1.0, (m, n, ok, worst)
    y = y_ref.copy()
    y[2, 5] = np.nan
    assert not o.check_linear(y, y_ref, bound)[0]
    ok, worst = o.check_linear(y_ref + 0.25 * allow, y_ref, bound)
    assert ok and worst == 0.25


def pin_linear_one_hot(o):
    """x = e_k picks column k of the dequantized weight (plus the bias)."""
    rng = np.random.default_rng(11)
    N, K = 9, 70
    W = rng.standard_normal((N, K)).astype(np.float32)
    q, s = o.quantize_rtn(W)
    codes = o.pack_nibbles(q)
    b = rng.standard_normal(N).astype(np.float32)
    w = o.dequantize(codes, s, K, "f32").astype(np.float64)
    for k in (0, 31, 32, 69):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y, bound = o.linear(x, codes, s, K, b)
        assert np.array_equal(y[0], w[:, k] + b.astype(np.float64))
        assert np.array_equal(bound[0], np.abs(w[:, k]))


def pin_linear_exact_rational(o):
    """Tiny random case against exact rational arithmetic built only from the
    packed bytes' definition (Python integers and Fractions, no NumPy math)."""
    rng = np.random.default_rng(5)
    M, N, K = 3, 5, 37
    vals = rng.integers(-8, 8, size=(N, K))
    codes = o.pack_nibbles(vals)
    s = rng.uniform(0.01, 2.0, size=(N, 2)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    b = rng.standard_normal(N).astype(np.float32)
    y, bound = o.linear(x, codes, s, K, b)
    for m in range(M):
        for n in range(N):
            acc = Fraction(float(b[n]))
            mag = Fraction(0)
            for k in range(K):
                byte = int(codes[n, k // 2])
                nib = (byte >> 4) if (k % 2) else (byte & 15)
                v = nib - 16 if nib >= 8 else nib
                wv = np.float32(v) * s[n, k // 32]  # one fp32 rounding, as the format says
                t = Fraction(float(x[m, k])) * Fraction(float(wv))
                acc += t
                mag += abs(t)
            assert abs(Fraction(y[m, n]) - acc) <= Fraction(1, 10**12) * (mag + 1)
            assert abs(Fraction(bound[m, n]) - mag) <= Fraction(1, 10**12) * (mag + 1)


def pin_asym_worked(o):
    g = read_golden("asym_worked_example.txt")
    K = int(g["width"][0])
    u = _ints(g["u"]).reshape(1, K)
    codes = o.pack_nibbles(u)
    assert np.array_equal(codes[0], _hex(g["bytes_hex"]))
    assert np.array_equal(o.unpack_unsigned(codes, K)[0], u[0])
    gi = _ints(g["g_idx"]).astype(np.int32)
    s = _floats(g["scales"]).astype(np.float32).reshape(1, -1)
    z = _ints(g["zeros"]).astype(np.int8).reshape(1, -1)
    w = o.dequantize_asym_gidx(codes, s, z, gi, K)
    assert np.array_equal(w[0].astype(np.float64), _floats(g["f32"])), w


def pin_asym_reduces_to_sym(o):
    """With g_idx = floor(k / 128), zero 8 and u = q + 8, the asymmetric dequant
    equals the symmetric one whose group-32 scales repeat each group-128 scale."""
    rng = np.random.default_rng(9)
    N, K = 6, 300
    q = rng.integers(-7, 8, size=(N, K))
    s128 = rng.uniform(0.001, 1.0, size=(N, math.ceil(K / 128))).astype(np.float32)
    s32 = np.repeat(s128, 4, axis=1)[:, : math.ceil(K / 32)]
    sym = o.dequantize(o.pack_nibbles(q), s32, K, "f32")
    gi = (np.arange(K) // 128).astype(np.int32)
    z = np.full(s128.shape, 8, np.int8)
    asym = o.dequantize_asym_gidx(o.pack_nibbles(q + 8), s128, z, gi, K)
    assert np.array_equal(sym, asym)


def pin_asym_permutation(o):
    """Permuting x's columns, the code columns and g_idx together leaves y
    unchanged (the act-order map only relabels columns)."""
    case = workloads.asym_case(M=3, N=8, K=256, group=64, seed=4)
    u, s, z = o.quantize_asym_minmax(case["W"], case["g_idx"], case["n_groups"])
    K = case["K"]
    y0, _ = o.linear_asym_gidx(case["x"], o.pack_nibbles(u), s, z, case["g_idx"], K, case["bias"])
    p = np.random.default_rng(1).permutation(K)
    y1, _ = o.linear_asym_gidx(case["x"][:, p], o.pack_nibbles(u[:, p]), s, z, case["g_idx"][p], K,
                               case["bias"])
    assert np.allclose(y0, y1, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# tests
# ---------------------------------------------------------------------------

def test_bf16_rne_matches_torch():
    pin_bf16_rne(O)


def test_f16_conversion_matches_torch():
    rng = np.random.default_rng(8)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 1000,
                        (rng.standard_normal(2000) * 1e-6).astype(np.float32)])
    codes = O.pack_nibbles(np.ones((1, v.size), np.int64))
    # dequantize(.., f16) of code 1 with scale v is fp16(v): compare to torch's RNE
    s = v.reshape(1, -1)[:, ::32].copy()
    got = O.dequantize(codes, np.abs(s) + np.float32(1e-30), v.size, "f16")
    ref = torch.from_numpy(np.repeat(np.abs(s) + np.float32(1e-30), 32, axis=1)[:, : v.size]).to(torch.float16)
    assert np.array_equal(got.view(np.uint16), ref.numpy().view(np.uint16))


def test_pack_worked_example():
    pin_pack_worked(O)


def test_unpack_brute_force_256():
    pin_unpack_brute_force(O)


def test_rtn_worked_example():
    pin_rtn_worked(O)


@pytest.mark.parametrize("shape,outliers", [((17, 1000), True), ((5, 33), False), ((3, 4095), False),
                                            ((64, 96), True)])
def test_rtn_invariants(shape, outliers):
    c = workloads.linear_case(21, 1, shape[0], shape[1], outliers=outliers)
    pin_rtn_invariants(O, c["W"])


def test_rtn_invariants_config1():
    pin_rtn_invariants(O, workloads.config1()["W"])


def test_rtn_extreme_values():
    W = np.array([[3.4e38, -3.4e38, 1.0, 0.0] + [0.0] * 28 + [1e-45, 0, 0, -1e-45, 7e-45]], np.float32)
    pin_rtn_invariants(O, W)
    q, s = O.quantize_rtn(W)
    assert s[0, 1] == O.FLOOR  # amax/7 of a subnormal group rounds below the floor


def test_rtn_rejects_bad_input():
    with pytest.raises(ValueError):
        O.quantize_rtn(np.zeros((0, 4), np.float32))
    with pytest.raises(ValueError):
        O.quantize_rtn(np.array([[1.0, np.nan]], np.float32))
    with pytest.raises(ValueError):
        O.quantize_rtn(np.array([[1.0, np.inf]], np.float32))
    with pytest.raises(ValueError):
        O.quantize_rtn(np.zeros(4, np.float32))


def test_dequant_worked_example():
    pin_dequant_worked(O)


def test_dequant_closed_form():
    pin_dequant_closed_form(O)


def test_linear_worked_example():
    pin_linear_worked(O)


def test_check_linear_acceptance():
    pin_check_linear(O)


def test_linear_one_hot():
    pin_linear_one_hot(O)


def test_linear_exact_rational():
    pin_linear_exact_rational(O)


def test_asym_worked_example():
    pin_asym_worked(O)


def test_asym_reduces_to_sym():
    pin_asym_reduces_to_sym(O)


def test_asym_permutation_invariance():
    pin_asym_permutation(O)


def test_asym_quantizer_shapes_data():
    """The asymmetric quantizer only shapes test data (parity unpinned); check the
    invariants that make its output a valid input: ranges, positivity and a
    reconstruction error of at most one scale step."""
    case = workloads.asym_case(M=1, N=16, K=512, group=128, seed=2)
    u, s, z = O.quantize_asym_minmax(case["W"], case["g_idx"], case["n_groups"])
    assert u.min() >= 0 and u.max() <= 15 and z.min() >= 0 and z.max() <= 15
    assert (s > 0).all() and np.isfinite(s).all()
    codes = O.pack_nibbles(u)
    assert O.validate_asym(codes, s, z, case["g_idx"], case["K"], case["n_groups"]) == "OK"
    w = O.dequantize_asym_gidx(codes, s, z, case["g_idx"], case["K"]).astype(np.float64)
    step = s[:, case["g_idx"]].astype(np.float64)
    assert (np.abs(w - case["W"]) <= step * (1 + 1e-6)).all()


def test_validate_rules():
    K, N = 5, 2
    codes = O.pack_nibbles(np.array([[1, -1, 7, -7, 0], [0, 1, 2, 3, 4]]))
    s = np.ones((N, 1), np.float32)
    assert O.validate(codes, s, K, 2) == "OK"
    assert O.validate(codes, s, K, 1) == "OK"
    assert O.validate(codes[:, :2], s, K, 2) == "SHAPE"
    assert O.validate(codes, np.ones((N, 2), np.float32), K, 2) == "SHAPE"
    assert O.validate(codes, s.astype(np.float64), K, 2) == "SHAPE"
    assert O.validate(codes, s, 0, 2) == "SHAPE"
    for bad in (0.0, -1.0, np.nan, np.inf):
        s2 = s.copy()
        s2[1, 0] = bad
        assert O.validate(codes, s2, K, 2) == "SCALE"
    c2 = codes.copy()
    c2[0, -1] |= 0x10
    assert O.validate(c2, s, K, 2) == "HIGH_NIBBLE"
    assert O.validate(codes, s, K, 3) == "VERSION"
    c3 = codes.copy()
    c3[1, 0] = 0x80
    assert O.validate(c3, s, K, 2) == "OK"
    assert O.validate(c3, s, K, 1) == "RESERVED_CODE"


def test_validate_asym_rules():
    K, N, G = 6, 2, 2
    codes = O.pack_nibbles(np.arange(12).reshape(N, K))
    s = np.ones((N, G), np.float32)
    z = np.full((N, G), 8, np.int8)
    gi = np.array([0, 1, 0, 1, 1, 0], np.int32)
    assert O.validate_asym(codes, s, z, gi, K, G) == "OK"
    assert O.validate_asym(codes, s, z, gi[:5], K, G) == "SHAPE"
    s2 = s.copy()
    s2[0, 0] = 0
    assert O.validate_asym(codes, s2, z, gi, K, G) == "SCALE"
    z2 = z.copy()
    z2[1, 1] = 16
    assert O.validate_asym(codes, s, z2, gi, K, G) == "ZERO"
    z2[1, 1] = -1
    assert O.validate_asym(codes, s, z2, gi, K, G) == "ZERO"
    gi2 = gi.copy()
    gi2[3] = 2
    assert O.validate_asym(codes, s, z, gi2, K, G) == "GIDX"
    gi2[3] = -1
    assert O.validate_asym(codes, s, z, gi2, K, G) == "GIDX"


def test_payload_bytes():
    """LoopQ payload_bytes = code bytes + 4 per scale; the decode shapes' figures."""
    assert O.payload_bytes(np.zeros((4096, 2048), np.uint8), np.zeros((4096, 128), np.float32)) == 10485760
    assert O.payload_bytes(np.zeros((14336, 2048), np.uint8), np.zeros((14336, 128), np.float32)) == 36700160
    assert O.payload_bytes(np.zeros((11008, 2048), np.uint8), np.zeros((11008, 32), np.float32),
                           np.zeros((11008, 32), np.int8), np.zeros(4096, np.int32)) == 24322048
