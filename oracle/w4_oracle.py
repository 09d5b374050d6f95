"""Plain NumPy oracle for the packed group-32 int4 weight format and the linear.

TEST INFRASTRUCTURE ONLY (see the package docstring). Every function is a direct
restatement of one definition on the source pages, written for a reader to check
by eye: loops over groups, whole-array NumPy element operations, and one library
matmul in float64 for the contraction. No blocking, fusion or reordering.

Sources (page title, then the function or section on it):

* LoopQ ``loopq/packed_weight.py`` -- ``PackedLoopQWeight`` (record layout),
  ``validate``, ``payload_bytes``, ``_dequantize_validated``, ``pack_weight``.
  This page fixes the storage contract: codes are uint8 ``[rows, ceil(width/2)]``
  with the even column in the low nibble, nibbles are two's complement (a value
  of 8 or more means value - 16), fp32 scales are ``[rows, ceil(width/32)]``,
  finite and positive, one scale per 32 consecutive columns, the last group
  truncated to the width; format version 1 forbids the nibble 8.
* gemma ``peft/_quantization_utils.py`` -- ``uniform_quantize``: abs-max scaling,
  round (NumPy/JAX ``round`` is round-half-to-even) and clip to the signed range.
* Keras ``layers/core/dense.py`` (int4 diff) -- ``_int4_build`` (sub-channel
  ``kernel_scale``/``kernel_zero`` per (group, output), ``g_idx`` mapping each
  input column to its group, default ``floor(k / block)``) and ``_int4_call``
  (dequantize with scale, zero and ``g_idx``, then matmul, then add the bias).
* PaddleNLP ``quantization/quantization_linear.py`` -- ``quant_weight_forward``
  (``weight_only_linear(x, weight, bias, weight_scale, weight_dtype,
  group_size)``): the fused weight-only linear y = x . dequant(W)^T + b.

Readings where the pages leave a step open are listed beside each function.
"""

from __future__ import annotations

import math

import numpy as np

GROUP = 32
"""Columns per scale in the symmetric format (LoopQ ``validate``: scales have
``ceil(width / 32)`` columns; ``_dequantize_validated`` repeats each scale 32 times)."""

FLOOR = np.float32(np.finfo(np.float32).tiny)
"""Positive floor on the RTN scale: the smallest normal fp32, 2**-126.

Reading: the rule only asks for "a positive floor". gemma's ``1e-6`` bounds a
*reciprocal* scale and does not carry over. FLT_MIN never changes a group whose
``amax / 7`` is a normal number, keeps every scale finite and positive (LoopQ
``validate``), and makes an all-zero group quantize to codes 0."""

QMAX = 7
"""Narrow signed range [-7, 7]: LoopQ format v1 reserves -8 (``validate``)."""

STATUS_NAMES = (
    "OK", "NULL", "SHAPE", "DTYPE", "NONFINITE", "SCALE", "HIGH_NIBBLE",
    "RESERVED_CODE", "VERSION", "GIDX", "ZERO", "UNSUPPORTED", "WORKSPACE",
    "TIMEOUT", "CUDA",
)
STATUS = {name: name for name in STATUS_NAMES}
"""Names of the outcomes ``validate`` can report (the oracle returns names, never
the library's integer codes)."""


# ---------------------------------------------------------------------------
# Floating-point format helpers (the oracle's own, pinned against torch in tests)
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 values to bfloat16 with round-to-nearest-even; return the bits.

    bfloat16 keeps the top 16 bits of the fp32 pattern. RNE adds half an ulp of
    the kept part (0x7FFF) plus the kept part's lowest bit (ties go to even) and
    truncates. NaN inputs keep their sign and become the quiet NaN 0x7FC0.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        sign = ((u >> np.uint64(16)) & np.uint64(0x8000)).astype(np.uint16)
        r = np.where(nan, sign | np.uint16(0x7FC0), r)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to fp32 (append 16 zero bits)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


# ---------------------------------------------------------------------------
# a1 + a2: RTN symmetric group-32 quantization and nibble packing
# ---------------------------------------------------------------------------

def quantize_rtn(W):
    """Round-to-nearest symmetric quantization, one fp32 scale per 32 columns.

    Follows LoopQ ``pack_weight`` for the checks and the order of steps, with the
    quantizer rule it imports (its body is not on the page) read as:

    for each row n and group g (columns ``32g .. min(32g+32, K)-1``):
      amax = max |w|                                  (exact)
      s    = max(fl32(amax / 7), FLOOR)               (IEEE fp32 divide)
      q    = clamp(round_half_even(fl32(w / s)), -7, 7)

    The rounding is gemma ``uniform_quantize``'s ``round`` (half to even); the
    clip range is narrowed to [-7, 7] because format v1 reserves -8 (LoopQ
    ``validate``). The scale multiplies the code (LoopQ ``_dequantize_validated``:
    ``values * scales``), the reciprocal of gemma's convention.

    Returns ``(q, scales)``: int8 ``[N, K]`` in [-7, 7] and fp32 ``[N, ceil(K/32)]``.
    Raises ValueError for an empty, non-2-D or non-finite W (``pack_weight``).
    """
    W = np.asarray(W)
    if W.ndim != 2 or min(W.shape) <= 0:
        raise ValueError("weight must be a nonempty matrix")
    W = W.astype(np.float32, copy=False)
    if not np.isfinite(W).all():
        raise ValueError("weight must be finite")
    N, K = W.shape
    G = math.ceil(K / GROUP)
    q = np.zeros((N, K), dtype=np.int8)
    scales = np.zeros((N, G), dtype=np.float32)
    seven = np.float32(QMAX)
    for g in range(G):
        lo, hi = GROUP * g, min(GROUP * g + GROUP, K)
        w = W[:, lo:hi]
        amax = np.max(np.abs(w), axis=1)
        s = np.maximum(amax / seven, FLOOR).astype(np.float32)
        t = (w / s[:, None]).astype(np.float32)
        qq = np.clip(np.rint(t), -QMAX, QMAX)
        q[:, lo:hi] = qq.astype(np.int8)
        scales[:, g] = s
    return q, scales


def quantize_rtn_channel(W):
    """Round-to-nearest symmetric quantization with one fp32 scale per output row.

    Keras ``quantize`` (int4 diff) on its per-channel branch (``block_size`` None or -1)
    uses ``AbsMaxQuantizer(axis=0, value_range=(-8, 7))``, one scale per output unit
    (``kernel_scale`` of shape ``(units,)``); the quantizer's body is not on the page.
    Reading, with the same rule as :func:`quantize_rtn` over the whole row instead of a
    32-column group and the Keras range:

      amax_n = max_k |w[n, k]|;   s_n = max(fl32(amax_n / 7), FLOOR)
      q      = clamp(round_half_even(fl32(w / s_n)), -8, 7)

    and the scale multiplies the code (LoopQ's convention; Keras divides by a multiplier
    ``7 / amax``, the same value up to rounding). With this scale |w / s| <= 7 up to the
    quotient's rounding, so the codes lie in [-7, 7] and are valid for format v1 too.

    Returns ``(q, scales)``: int8 ``[N, K]`` and fp32 ``[N]``. Raises ValueError for an
    empty, non-2-D or non-finite W.
    """
    W = np.asarray(W)
    if W.ndim != 2 or min(W.shape) <= 0:
        raise ValueError("weight must be a nonempty matrix")
    W = W.astype(np.float32, copy=False)
    if not np.isfinite(W).all():
        raise ValueError("weight must be finite")
    amax = np.max(np.abs(W), axis=1)
    s = np.maximum(amax / np.float32(QMAX), FLOOR).astype(np.float32)
    t = (W / s[:, None]).astype(np.float32)
    q = np.clip(np.rint(t), -8, 7).astype(np.int8)
    return q, s


def expand_channel_scales(scales_channel, K: int) -> np.ndarray:
    """Per-row scales ``[N]`` as the group layout ``[N, ceil(K/32)]`` (every group of a row
    carries the row's scale): a per-channel weight is then a packed group-32 weight."""
    s = np.asarray(scales_channel, dtype=np.float32).reshape(-1, 1)
    return np.repeat(s, math.ceil(K / GROUP), axis=1)


def pack_nibbles(values) -> np.ndarray:
    """Pack 4-bit values two per byte along the width, even column in the low nibble.

    LoopQ ``pack_weight``: ``unsigned = integers & 15``; an odd width is padded
    with one zero column; ``byte = unsigned[:, 0::2] | unsigned[:, 1::2] << 4``.
    Works for signed codes in [-8, 7] and unsigned codes in [0, 15] alike.
    """
    v = np.asarray(values)
    if v.ndim != 2:
        raise ValueError("values must be 2-D")
    u = (v.astype(np.int16) & 15).astype(np.uint8)
    if u.shape[1] % 2:
        u = np.concatenate([u, np.zeros((u.shape[0], 1), np.uint8)], axis=1)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def unpack_unsigned(codes, K: int) -> np.ndarray:
    """Nibbles as unsigned values in [0, 15], interleaved low-then-high and
    truncated to the width K (LoopQ ``_dequantize_validated``: ``stack((codes & 15,
    codes >> 4), -1).flatten(-2)[:, :width]``)."""
    c = np.asarray(codes, dtype=np.uint8)
    pairs = np.stack((c & 15, c >> 4), axis=-1).reshape(c.shape[0], -1)
    return pairs[:, :K].astype(np.int16)


def unpack_signed(codes, K: int) -> np.ndarray:
    """Two's-complement nibbles: a value of 8 or more stands for value - 16
    (LoopQ ``_dequantize_validated``: ``where(values >= 8, values - 16, values)``)."""
    v = unpack_unsigned(codes, K)
    return np.where(v >= 8, v - 16, v).astype(np.int16)


# ---------------------------------------------------------------------------
# a3 + a4: dequantization
# ---------------------------------------------------------------------------

def dequantize(codes, scales, K: int, out_dtype: str = "f32"):
    """Dequantize packed codes: fp32 product ``value * scale``, then the output
    dtype (LoopQ ``_dequantize_validated``: ``(values * scales).to(dtype)`` with
    ``scales.repeat_interleave(32)[:, :width]``).

    The product is one IEEE fp32 multiply; the conversion to bf16/f16 then rounds
    to nearest even (``Tensor.to``); f64 is an exact widening. bf16 results are
    returned as uint16 bit patterns.
    """
    v = unpack_signed(codes, K).astype(np.float32)
    s = np.repeat(np.asarray(scales, dtype=np.float32), GROUP, axis=1)[:, :K]
    w32 = (v * s).astype(np.float32)
    if out_dtype == "f32":
        return w32
    if out_dtype == "bf16":
        return f32_to_bf16_bits(w32)
    if out_dtype == "f16":
        return w32.astype(np.float16)
    if out_dtype == "f64":
        return w32.astype(np.float64)
    raise ValueError("unsupported output dtype")


# ---------------------------------------------------------------------------
# a5: the fused linear, symmetric format
# ---------------------------------------------------------------------------

def linear(x, codes, scales, K: int, bias=None):
    """Reference for ``y = x . dequant(W)^T + b`` in float64.

    Keras ``_int4_call`` dequantizes the kernel, multiplies, then adds the bias;
    PaddleNLP ``quant_weight_forward`` fuses the same into ``weight_only_linear``.
    Here: ``w = dequantize(..., "f32")`` (the exact fp32 dequantized weight),
    ``y[m, n] = sum_k x[m, k] * w[n, k] + b[n]`` in float64, and the error scale
    ``bound[m, n] = sum_k |x[m, k] * w[n, k]|`` that the tolerance multiplies.

    ``x`` holds the activation values as fp32 (bf16 activations widen exactly).
    Returns ``(y_ref, bound)``, both float64 ``[M, N]``.
    """
    x64 = np.asarray(x, dtype=np.float32).astype(np.float64)
    w64 = dequantize(codes, scales, K, "f32").astype(np.float64)
    y = x64 @ w64.T
    bound = np.abs(x64) @ np.abs(w64).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    return y, bound


def check_linear(y_gpu, y_ref, bound, rtol: float = 4e-3, atol: float = 1e-6):
    """Per-element acceptance ``|y - y_ref| <= rtol * bound + atol``.

    Returns ``(ok, worst)`` where ``worst`` is the largest ratio of the error to
    its allowance (<= 1 means every element passed)."""
    y = np.asarray(y_gpu, dtype=np.float64)
    err = np.abs(y - y_ref)
    allow = rtol * bound + atol
    worst = float(np.max(err / allow)) if err.size else 0.0
    return bool(np.all(err <= allow)), worst


# ---------------------------------------------------------------------------
# backward of the linear with respect to its input
# ---------------------------------------------------------------------------

def linear_backward_x(dy, codes, scales, K: int):
    """Reference for the input gradient ``dx = dy . dequant(W)`` in float64.

    Keras ``_int4_call``'s ``grad_fn`` returns ``matmul(upstream, transpose(float_kernel))``
    with the kernel stored ``[in, out]``; PaddleNLP ``QuantizationLinearFunc.backward``
    returns ``matmul(grad_output, qdq_weight.T)``. With the packed weight stored ``[N, K]``
    (rows = output features) both are ``dx[m, k] = sum_n dy[m, n] * w[n, k]``, ``w`` the
    exact fp32 dequantized weight (reading: the pages cast it to the compute dtype first;
    the tolerance covers that rounding). Also ``bound[m, k] = sum_n |dy[m, n] * w[n, k]|``.

    ``dy`` holds the upstream gradient values as fp32 (bf16 gradients widen exactly).
    Returns ``(dx_ref, bound)``, both float64 ``[M, K]``.
    """
    dy64 = np.asarray(dy, dtype=np.float32).astype(np.float64)
    w64 = dequantize(codes, scales, K, "f32").astype(np.float64)
    return dy64 @ w64, np.abs(dy64) @ np.abs(w64)


# ---------------------------------------------------------------------------
# LoRA merge: dequantize, add the low-rank update, re-quantize, re-pack
# ---------------------------------------------------------------------------

def lora_merge(codes, scales, K: int, lora_b_t, lora_a_t, alpha_over_rank):
    """Merge a LoRA update into a packed weight and re-quantize it.

    Keras ``Dense`` (int4 diff), the merged-kernel helper: Step 1 dequantizes the kernel,
    Step 2 adds ``(lora_alpha / lora_rank) * matmul(lora_kernel_a, lora_kernel_b)`` in the
    float domain, Step 3 re-quantizes and packs. With the weight stored ``[N, K]`` the
    update is ``delta[n, k] = c * sum_j b[n, j] * a[j, k]`` with ``b = lora_kernel_b^T``
    ``[N, r]``, ``a = lora_kernel_a^T`` ``[r, K]`` and ``c = alpha / rank``.

    Reading (fp32 throughout, each step rounded, in this order, so that the re-quantized
    codes are a function of the inputs alone):
      w      = fl32(q * s)                                   (the dequantized weight)
      t      = 0;  for j = 0 .. r-1:  t = fl32(t + fl32(b[n, j] * a[j, k]))
      w'     = fl32(w + fl32(c * t))
    then :func:`quantize_rtn` on ``w'`` (this library's group-32 rule; Keras re-quantizes
    into its own layouts). Returns ``(q', scales')`` as :func:`quantize_rtn`.
    """
    w = dequantize(codes, scales, K, "f32")
    b = np.asarray(lora_b_t, dtype=np.float32)
    a = np.asarray(lora_a_t, dtype=np.float32)
    if b.shape[0] != w.shape[0] or a.shape[1] != K or b.shape[1] != a.shape[0]:
        raise ValueError("lora_b_t must be [N, r] and lora_a_t [r, K]")
    t = np.zeros_like(w, dtype=np.float32)
    for j in range(b.shape[1]):
        prod = (b[:, j:j + 1] * a[j:j + 1, :]).astype(np.float32)
        t = (t + prod).astype(np.float32)
    merged = (w + (np.float32(alpha_over_rank) * t).astype(np.float32)).astype(np.float32)
    return quantize_rtn(merged)


# ---------------------------------------------------------------------------
# a6: asymmetric sub-channel variant with act-order g_idx
# ---------------------------------------------------------------------------

def dequantize_asym_gidx(codes, scales, zeros, g_idx, K: int) -> np.ndarray:
    """Asymmetric dequantization through a column-to-group map.

    Keras ``_int4_call`` (sub-channel branch) calls ``dequantize_with_sz_map``
    with the kernel, ``kernel_scale``, ``kernel_zero`` and ``g_idx``; the helper's
    body is not on the page. Reading: the zero point is in code units and is
    subtracted before the scale, ``w[n, k] = fl32((u[n, k] - z[n, g]) * s[n, g])``
    with ``g = g_idx[k]`` and ``u`` the *unsigned* nibble in [0, 15]. The layout
    follows the packed contract: rows are output features, so scale and zero are
    ``[N, n_groups]`` (the transpose of Keras's ``[n_groups, out]``).
    """
    u = unpack_unsigned(codes, K)
    gi = np.asarray(g_idx).astype(np.int64)
    s = np.asarray(scales, dtype=np.float32)[:, gi]
    z = np.asarray(zeros).astype(np.int16)[:, gi]
    return ((u - z).astype(np.float32) * s).astype(np.float32)


def linear_asym_gidx(x, codes, scales, zeros, g_idx, K: int, bias=None):
    """``y = x . dequant_asym(W)^T + b`` in float64, with its error scale (as
    ``linear``)."""
    x64 = np.asarray(x, dtype=np.float32).astype(np.float64)
    w64 = dequantize_asym_gidx(codes, scales, zeros, g_idx, K).astype(np.float64)
    y = x64 @ w64.T
    bound = np.abs(x64) @ np.abs(w64).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    return y, bound


def quantize_asym_minmax(W, g_idx, n_groups: int):
    """Asymmetric min-max quantizer used only to *shape* synthetic asymmetric data.

    Parity unpinned: Keras ``quantize`` calls ``abs_max_quantize_grouped_with_zero_point``
    whose body is not on the page. Reading, per row n and group g (the columns k
    with ``g_idx[k] == g``): ``lo = min(min w, 0)``, ``hi = max(max w, 0)``,
    ``s = max(fl32((hi - lo) / 15), FLOOR)``, ``z = clamp(rne(-lo / s), 0, 15)``,
    ``u = clamp(rne(w / s) + z, 0, 15)``. The library never runs this step; both
    sides of the parity tests consume the same ``u``, ``z``, ``s``.

    Returns ``(u uint8 [N, K], scales f32 [N, n_groups], zeros int8 [N, n_groups])``.
    """
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    gi = np.asarray(g_idx).astype(np.int64)
    u = np.zeros((N, K), dtype=np.uint8)
    scales = np.zeros((N, n_groups), dtype=np.float32)
    zeros = np.zeros((N, n_groups), dtype=np.int8)
    fifteen = np.float32(15)
    for g in range(n_groups):
        cols = np.nonzero(gi == g)[0]
        if cols.size == 0:
            scales[:, g] = FLOOR
            continue
        w = W[:, cols]
        lo = np.minimum(w.min(axis=1), np.float32(0))
        hi = np.maximum(w.max(axis=1), np.float32(0))
        s = np.maximum((hi - lo) / fifteen, FLOOR).astype(np.float32)
        z = np.clip(np.rint((-lo / s).astype(np.float32)), 0, 15)
        t = np.rint((w / s[:, None]).astype(np.float32)) + z[:, None]
        u[:, cols] = np.clip(t, 0, 15).astype(np.uint8)
        scales[:, g] = s
        zeros[:, g] = z.astype(np.int8)
    return u, scales, zeros


# ---------------------------------------------------------------------------
# Content checks and the payload metric
# ---------------------------------------------------------------------------

def validate(codes, scales, K: int, format_version: int = 2, N: int | None = None) -> str:
    """LoopQ ``PackedLoopQWeight.validate`` for one packed weight; returns the name
    of the first rule that fails, in the page's order, or ``"OK"``.

    shape positive -> code shape/dtype -> scale shape/dtype -> scales finite and
    positive -> unused high nibble of an odd width is zero -> version in {1, 2} ->
    (v1 only) no nibble equal to 8. The output-dtype rule belongs to the call that
    names a dtype and is not checked here.
    """
    codes = np.asarray(codes)
    scales = np.asarray(scales)
    if N is None:
        N = codes.shape[0] if codes.ndim == 2 else 0
    if N <= 0 or K <= 0:
        return "SHAPE"
    if codes.dtype != np.uint8 or codes.shape != (N, math.ceil(K / 2)):
        return "SHAPE"
    if scales.dtype != np.float32 or scales.shape != (N, math.ceil(K / GROUP)):
        return "SHAPE"
    if not (np.isfinite(scales).all() and (scales > 0).all()):
        return "SCALE"
    if K % 2 and (codes[:, -1] >> 4).any():
        return "HIGH_NIBBLE"
    if format_version not in (1, 2):
        return "VERSION"
    if format_version == 1 and (((codes & 15) == 8).any() or ((codes >> 4) == 8).any()):
        return "RESERVED_CODE"
    return "OK"


def validate_asym(codes, scales, zeros, g_idx, K: int, n_groups: int) -> str:
    """Checks for the asymmetric variant, in the same spirit as ``validate``:
    shapes, scales finite and positive, the odd-width pad nibble zero, zero points
    in the unsigned code range [0, 15] (Keras stores them as int8), and every
    ``g_idx`` entry naming an existing group."""
    codes = np.asarray(codes)
    scales = np.asarray(scales)
    zeros = np.asarray(zeros)
    g_idx = np.asarray(g_idx)
    N = codes.shape[0] if codes.ndim == 2 else 0
    if N <= 0 or K <= 0 or n_groups <= 0:
        return "SHAPE"
    if codes.dtype != np.uint8 or codes.shape != (N, math.ceil(K / 2)):
        return "SHAPE"
    if scales.shape != (N, n_groups) or zeros.shape != (N, n_groups) or g_idx.shape != (K,):
        return "SHAPE"
    if not (np.isfinite(scales).all() and (scales > 0).all()):
        return "SCALE"
    if K % 2 and (codes[:, -1] >> 4).any():
        return "HIGH_NIBBLE"
    if ((zeros < 0) | (zeros > 15)).any():
        return "ZERO"
    if ((g_idx < 0) | (g_idx >= n_groups)).any():
        return "GIDX"
    return "OK"


def payload_bytes(codes, scales, zeros=None, g_idx=None) -> int:
    """Tensor payload of a packed weight (LoopQ ``payload_bytes``: code bytes plus
    four bytes per scale), extended for the asymmetric variant by one byte per
    zero point and four per ``g_idx`` entry."""
    n = int(np.asarray(codes).size) + 4 * int(np.asarray(scales).size)
    if zeros is not None:
        n += int(np.asarray(zeros).size)
    if g_idx is not None:
        n += 4 * int(np.asarray(g_idx).size)
    return n
