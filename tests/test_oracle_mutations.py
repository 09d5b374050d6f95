"""Each test plants one plausible mistake in the CPU oracle (monkeypatched, on the
CPU) and checks that at least one pin catches it. This shows the pins are strong
enough to hold the oracle in place: a dropped term, a wrong sign, index or
rounding mode, or a swapped operand fails a pin."""

import math

import numpy as np
import pytest

import oracle.w4_oracle as O
import test_oracle_pins as P
import workloads


def _fails(pin, *args):
    with pytest.raises(AssertionError):
        pin(O, *args)


def test_mutant_nibble_order_swapped(monkeypatch):
    def pack_odd_low(values):
        u = (np.asarray(values).astype(np.int16) & 15).astype(np.uint8)
        if u.shape[1] % 2:
            u = np.concatenate([u, np.zeros((u.shape[0], 1), np.uint8)], axis=1)
        return (u[:, 1::2] | (u[:, 0::2] << 4)).astype(np.uint8)
    monkeypatch.setattr(O, "pack_nibbles", pack_odd_low)
    _fails(P.pin_pack_worked)


def test_mutant_sign_threshold(monkeypatch):
    orig = O.unpack_unsigned

    def unpack_signed_bad(codes, K):
        v = orig(codes, K)
        return np.where(v >= 7, v - 16, v).astype(np.int16)
    monkeypatch.setattr(O, "unpack_signed", unpack_signed_bad)
    _fails(P.pin_unpack_brute_force)


def test_mutant_round_half_away(monkeypatch):
    def rint_away(t):
        return np.sign(t) * np.floor(np.abs(t) + 0.5)
    monkeypatch.setattr(O.np, "rint", rint_away)
    try:
        _fails(P.pin_rtn_worked)
    finally:
        monkeypatch.undo()


def test_mutant_scale_divisor(monkeypatch):
    monkeypatch.setattr(O, "QMAX", 8)
    _fails(P.pin_rtn_worked)


def test_mutant_scale_reciprocal(monkeypatch):
    """gemma's multiplier convention (dequant = q / scale) instead of q * scale."""
    def dequant_div(codes, scales, K, out_dtype="f32"):
        v = O.unpack_signed(codes, K).astype(np.float32)
        s = np.repeat(np.asarray(scales, np.float32), 32, axis=1)[:, :K]
        w = (v / s).astype(np.float32)
        return O.f32_to_bf16_bits(w) if out_dtype == "bf16" else w.astype(
            {"f32": np.float32, "f16": np.float16, "f64": np.float64}[out_dtype])
    monkeypatch.setattr(O, "dequantize", dequant_div)
    _fails(P.pin_dequant_worked)


def test_mutant_scale_group_index(monkeypatch):
    def dequant_shift(codes, scales, K, out_dtype="f32"):
        v = O.unpack_signed(codes, K).astype(np.float32)
        s = np.repeat(np.roll(np.asarray(scales, np.float32), 1, axis=1), 32, axis=1)[:, :K]
        return (v * s).astype(np.float32)
    monkeypatch.setattr(O, "dequantize", dequant_shift)
    _fails(P.pin_dequant_closed_form)


def test_mutant_group_size_64(monkeypatch):
    monkeypatch.setattr(O, "GROUP", 64)
    _fails(P.pin_rtn_worked)


def test_mutant_bf16_truncation(monkeypatch):
    def trunc(a):
        return (np.ascontiguousarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    monkeypatch.setattr(O, "f32_to_bf16_bits", trunc)
    _fails(P.pin_bf16_rne)


def test_mutant_dropped_bias(monkeypatch):
    orig = O.linear

    def linear_nobias(x, codes, scales, K, bias=None):
        return orig(x, codes, scales, K, None)
    monkeypatch.setattr(O, "linear", linear_nobias)
    _fails(P.pin_linear_worked)


def test_mutant_transposed_weight(monkeypatch):
    """Contracting over the wrong weight axis (rows instead of columns)."""
    def linear_T(x, codes, scales, K, bias=None):
        w = O.dequantize(codes, scales, K, "f32").astype(np.float64)
        x64 = np.asarray(x, np.float64)
        wt = w.T.reshape(w.shape)  # data read in transposed order
        y = x64 @ wt.T
        if bias is not None:
            y = y + np.asarray(bias, np.float64)
        return y, np.abs(x64) @ np.abs(wt).T
    monkeypatch.setattr(O, "linear", linear_T)
    _fails(P.pin_linear_exact_rational)


def test_mutant_bound_without_abs(monkeypatch):
    def linear_signed_bound(x, codes, scales, K, bias=None):
        w = O.dequantize(codes, scales, K, "f32").astype(np.float64)
        x64 = np.asarray(x, np.float64)
        y = x64 @ w.T + (0 if bias is None else np.asarray(bias, np.float64))
        return y, x64 @ w.T
    monkeypatch.setattr(O, "linear", linear_signed_bound)
    _fails(P.pin_linear_worked)


def test_mutant_asym_zero_added(monkeypatch):
    def deq(codes, scales, zeros, g_idx, K):
        u = O.unpack_unsigned(codes, K)
        gi = np.asarray(g_idx).astype(np.int64)
        return ((u + np.asarray(zeros).astype(np.int16)[:, gi]).astype(np.float32)
                * np.asarray(scales, np.float32)[:, gi]).astype(np.float32)
    monkeypatch.setattr(O, "dequantize_asym_gidx", deq)
    _fails(P.pin_asym_worked)


def test_mutant_asym_ignores_gidx(monkeypatch):
    def deq(codes, scales, zeros, g_idx, K):
        u = O.unpack_unsigned(codes, K)
        G = np.asarray(scales).shape[1]
        gi = (np.arange(K) * G // K).astype(np.int64)  # contiguous groups
        return ((u - np.asarray(zeros).astype(np.int16)[:, gi]).astype(np.float32)
                * np.asarray(scales, np.float32)[:, gi]).astype(np.float32)
    monkeypatch.setattr(O, "dequantize_asym_gidx", deq)
    _fails(P.pin_asym_worked)


def test_mutant_amax_over_padding(monkeypatch):
    """Taking the last group's amax over 32 columns read past the width (here:
    wrapping into the row's first columns) changes the partial group's scale."""
    orig = O.quantize_rtn

    def q_bad(W):
        W = np.asarray(W, np.float32)
        K = W.shape[1]
        pad = (-K) % 32
        Wp = np.concatenate([W, W[:, :pad]], axis=1) if pad else W
        q, s = orig(Wp)
        return q[:, :K], s[:, : math.ceil(K / 32)]
    monkeypatch.setattr(O, "quantize_rtn", q_bad)
    _fails(P.pin_rtn_worked)


def _check_linear_variant(any_=False, swap=False, strict=False, signed=False):
    def check(y_gpu, y_ref, bound, rtol=4e-3, atol=1e-6):
        y = np.asarray(y_gpu, np.float64)
        err = (y - y_ref) if signed else np.abs(y - y_ref)
        allow = (atol * bound + rtol) if swap else (rtol * bound + atol)
        passed = (err < allow) if strict else (err <= allow)
        worst = float(np.max(err / allow)) if err.size else 0.0
        return bool(np.any(passed) if any_ else np.all(passed)), worst
    return check


@pytest.mark.parametrize("kind", ["any_", "swap", "strict", "signed"])
def test_mutant_check_linear(monkeypatch, kind):
    """An acceptance test that passes if any element passes, swaps the relative and
    absolute terms, rejects an error equal to its allowance, or forgets the absolute
    value each fails the acceptance pin."""
    monkeypatch.setattr(O, "check_linear", _check_linear_variant(**{kind: True}))
    _fails(P.pin_check_linear)


def test_pins_pass_unmutated():
    P.pin_rtn_invariants(O, workloads.linear_case(1, 1, 8, 100)["W"])
