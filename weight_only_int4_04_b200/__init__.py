"""Python binding of libw4: group-wise 4-bit weight-only quantization and the
dequantize-fused linear for one B200 (sm_100a).

Argument marshalling only: every step runs in the CUDA kernels of ``libw4.so`` behind the
C ABI in ``include/w4.h``. PyTorch provides device memory and the current stream. There is
no CPU fallback: importing this package without the built library raises ImportError, and
every call requires CUDA tensors.

Packed format (page "loopq/packed_weight.py", PackedLoopQWeight): ``codes`` uint8
``[N, ceil(K/2)]`` (even column in the low nibble, two's-complement nibbles) and ``scales``
float32 ``[N, ceil(K/32)]``.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw4.so")

STATUS = {
    0: "OK", 1: "NULL", 2: "SHAPE", 3: "DTYPE", 4: "NONFINITE", 5: "SCALE", 6: "HIGH_NIBBLE",
    7: "RESERVED_CODE", 8: "VERSION", 9: "GIDX", 10: "ZERO", 11: "UNSUPPORTED", 12: "WORKSPACE",
    13: "TIMEOUT", 14: "CUDA",
}
DTYPES = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2, torch.float64: 3}

EXPORTS = (
    "w4_quantize_rtn", "w4_dequantize", "w4_linear", "w4_linear_workspace_bytes", "w4_linear_asym_workspace_bytes",
    "w4_asym_prepare", "w4_linear_asym_gidx", "w4_linear_asym_gidx_noalloc", "w4_validate", "w4_validate_asym",
    "w4_set_weight_prefetch", "w4_device_error", "w4_last_cuda_error", "w4_status_string", "w4_version",
    "w4_dequantize_q4_0", "w4_linear_q4_0", "w4_linear_backward_x_workspace_bytes", "w4_linear_backward_x",
    "w4_quantize_rtn_channel", "w4_expand_channel_scales", "w4_lora_merge", "w4_selftest_wait_timeout",
    "w4_last_linear_kernel", "w4_linear_channel_workspace_bytes", "w4_linear_channel", "w4_q4_0_to_group32",
)

_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "w4_quantize_rtn": [_vp, _i64, _i64, _vp, _vp, _vp, _vp],
    "w4_dequantize": [_vp, _vp, _i64, _i64, _i32, _i32, _vp, _vp],
    "w4_linear": [_vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _i32, _vp, _sz, _vp],
    "w4_linear_workspace_bytes": [_i64, _i64, _i64],
    "w4_linear_asym_workspace_bytes": [_i64, _i64, _i64, _i64],
    "w4_asym_prepare": [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _vp],
    "w4_linear_asym_gidx": [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _i32, _vp, _sz,
                            _vp],
    "w4_linear_asym_gidx_noalloc": [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp, _i32, _vp],
    "w4_validate": [_vp, _vp, _i64, _i64, _i32, _vp],
    "w4_validate_asym": [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp],
    "w4_set_weight_prefetch": [_i32],
    "w4_device_error": [],
    "w4_last_cuda_error": [],
    "w4_status_string": [_i32],
    "w4_version": [],
    "w4_dequantize_q4_0": [_vp, _i64, _i64, _i32, _vp, _vp],
    "w4_q4_0_to_group32": [_vp, _i64, _i64, _vp, _vp, _vp],
    "w4_linear_q4_0": [_vp, _i64, _vp, _i64, _i64, _vp, _vp, _i32, _vp],
    "w4_linear_backward_x_workspace_bytes": [_i64, _i64, _i64],
    "w4_linear_backward_x": [_vp, _i64, _vp, _vp, _i64, _i64, _vp, _i32, _vp, _sz, _vp],
    "w4_quantize_rtn_channel": [_vp, _i64, _i64, _vp, _vp, _vp, _vp],
    "w4_expand_channel_scales": [_vp, _i64, _i64, _vp, _vp],
    "w4_lora_merge": [_vp, _vp, _i64, _i64, _vp, _vp, _i64, ctypes.c_float, _vp, _vp, _vp, _vp],
    "w4_selftest_wait_timeout": [ctypes.c_uint64, _vp],
    "w4_last_linear_kernel": [],
    "w4_linear_channel_workspace_bytes": [_i64, _i64, _i64],
    "w4_linear_channel": [_vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _i32, _vp, _sz, _vp],
}
_lib = None


def _load():
    """Load libw4.so on first use; raise loudly if it was never built (no CPU fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m weight_only_int4_04_b200.build` "
                "(there is no CPU fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(handle, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        handle.w4_linear_workspace_bytes.restype = ctypes.c_size_t
        handle.w4_linear_asym_workspace_bytes.restype = ctypes.c_size_t
        handle.w4_linear_backward_x_workspace_bytes.restype = ctypes.c_size_t
        handle.w4_linear_channel_workspace_bytes.restype = ctypes.c_size_t
        handle.w4_status_string.restype = ctypes.c_char_p
        handle.w4_last_linear_kernel.restype = ctypes.c_char_p
        _lib = handle
    return _lib


def __getattr__(name):
    # `lib` is the loaded library; resolved lazily so that the build module can be imported
    # (and run) before the library exists.
    if name == "lib":
        return _load()
    raise AttributeError(name)


class W4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        msg = _load().w4_status_string(status).decode()
        if self.name == "CUDA":
            msg += f" (cudaError {_load().w4_last_cuda_error()})"
        super().__init__(f"{where}: {self.name}: {msg}")


def _check(status: int, where: str):
    if status != 0:
        raise W4Error(status, where)


def _ptr(t):
    # ctypes converts a plain int for a c_void_p argument; no wrapper object per pointer
    return None if t is None else t.data_ptr()


try:
    _raw_stream = torch._C._cuda_getCurrentRawStream  # the current stream's handle as an int
except AttributeError:  # pragma: no cover - older torch
    _raw_stream = None


def _stream():
    """Handle of the current device's current CUDA stream."""
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("w4: tensors must be contiguous CUDA tensors (no CPU fallback)")


def quantize_rtn(W: torch.Tensor, status: torch.Tensor | None = None, out=None):
    """RTN symmetric group-32 quantization of fp32 ``W [N, K]`` -> ``(codes, scales)``.

    With ``status`` (an int32 CUDA tensor of one element, zeroed by the caller) the call
    stays asynchronous and a non-finite W sets it to the NONFINITE code; without it the
    call synchronizes and raises ``W4Error`` for a non-finite W. ``out``: optional
    preallocated ``(codes uint8 [N, ceil(K/2)], scales float32 [N, ceil(K/32)])``."""
    _need_cuda(W, status)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    N, K = W.shape
    if out is None:
        codes = torch.empty((N, (K + 1) // 2), dtype=torch.uint8, device=W.device)
        scales = torch.empty((N, (K + 31) // 32), dtype=torch.float32, device=W.device)
    else:
        codes, scales = out
        _need_cuda(codes, scales)
        if codes.shape != (N, (K + 1) // 2) or scales.shape != (N, (K + 31) // 32) or \
                codes.dtype != torch.uint8 or scales.dtype != torch.float32:
            raise ValueError("out must be (uint8 [N, ceil(K/2)], float32 [N, ceil(K/32)])")
    _check(_load().w4_quantize_rtn(_ptr(W), N, K, _ptr(codes), _ptr(scales), _ptr(status), _stream()),
           "w4_quantize_rtn")
    return codes, scales


def quantize_rtn_channel(W: torch.Tensor, status: torch.Tensor | None = None):
    """Per-channel RTN quantization of fp32 ``W [N, K]`` -> ``(codes uint8 [N, ceil(K/2)],
    scales float32 [N])``, one scale per row (``status`` as in :func:`quantize_rtn`)."""
    _need_cuda(W, status)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    N, K = W.shape
    codes = torch.empty((N, (K + 1) // 2), dtype=torch.uint8, device=W.device)
    scales = torch.empty((N,), dtype=torch.float32, device=W.device)
    _check(_load().w4_quantize_rtn_channel(_ptr(W), N, K, _ptr(codes), _ptr(scales), _ptr(status), _stream()),
           "w4_quantize_rtn_channel")
    return codes, scales


def lora_merge(codes: torch.Tensor, scales: torch.Tensor, K: int, lora_b_t: torch.Tensor | None,
               lora_a_t: torch.Tensor | None, alpha_over_rank: float, out=None, status: torch.Tensor | None = None):
    """Merge ``alpha_over_rank * lora_b_t [N, r] . lora_a_t [r, K]`` into the packed weight and
    re-quantize; returns ``(codes', scales')`` (``out`` may be ``(codes, scales)``: in place)."""
    _need_cuda(codes, scales, lora_b_t, lora_a_t, status)
    N = codes.shape[0]
    r = 0 if lora_b_t is None else lora_b_t.shape[1]
    if r and (lora_b_t.dtype != torch.float32 or lora_a_t is None or lora_a_t.dtype != torch.float32 or
              lora_b_t.shape != (N, r) or lora_a_t.shape != (r, K)):
        raise ValueError("lora_b_t must be float32 [N, r] and lora_a_t float32 [r, K]")
    if out is None:
        out = (torch.empty_like(codes), torch.empty_like(scales))
    co, so = out
    _need_cuda(co, so)
    _check(_load().w4_lora_merge(_ptr(codes), _ptr(scales), N, K, _ptr(lora_b_t), _ptr(lora_a_t), r,
                                 float(alpha_over_rank), _ptr(co), _ptr(so), _ptr(status), _stream()),
           "w4_lora_merge")
    return co, so


def linear_channel(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, K: int | None = None,
                   bias: torch.Tensor | None = None, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None) -> torch.Tensor:
    """``y = x . dequant(W)^T + bias`` for a per-channel weight (``scales`` float32 ``[N]``)."""
    _need_cuda(x, codes, scales, bias, out, workspace)
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    if scales.dtype != torch.float32 or scales.dim() != 1:
        raise ValueError("scales must be a 1-D float32 tensor (one per row)")
    M, Kx = x.shape
    K = Kx if K is None else K
    if K != Kx:
        raise ValueError("x width does not match K")
    N = codes.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    need = int(_load().w4_linear_channel_workspace_bytes(M, N, K))
    ws, wsb = _workspace(M, N, K, x.device, workspace, need)
    _check(_load().w4_linear_channel(_ptr(x), M, _ptr(codes), _ptr(scales), N, K, _ptr(bias), _ptr(out),
                                     DTYPES[out.dtype], _ptr(ws), wsb, _stream()), "w4_linear_channel")
    return out


def expand_channel_scales(scales: torch.Tensor, K: int) -> torch.Tensor:
    """Per-row scales ``[N]`` -> the group layout ``[N, ceil(K/32)]`` every other call reads."""
    _need_cuda(scales)
    if scales.dtype != torch.float32 or scales.dim() != 1:
        raise ValueError("scales must be a 1-D float32 tensor")
    N = scales.shape[0]
    out = torch.empty((N, (K + 31) // 32), dtype=torch.float32, device=scales.device)
    _check(_load().w4_expand_channel_scales(_ptr(scales), N, K, _ptr(out), _stream()), "w4_expand_channel_scales")
    return out


def dequantize(codes: torch.Tensor, scales: torch.Tensor, K: int, out_dtype=torch.float32,
               format_version: int = 2, out: torch.Tensor | None = None) -> torch.Tensor:
    """Dense ``[N, K]`` weight of ``out_dtype`` (bf16, f16, f32 or f64)."""
    _need_cuda(codes, scales, out)
    N = codes.shape[0]
    if out_dtype not in DTYPES:
        raise ValueError("unsupported output dtype")
    if out is None:
        out = torch.empty((N, K), dtype=out_dtype, device=codes.device)
    _check(_load().w4_dequantize(_ptr(codes), _ptr(scales), N, K, format_version, DTYPES[out_dtype], _ptr(out),
                             _stream()), "w4_dequantize")
    return out


def _q4_0_shape(blocks: torch.Tensor, K: int) -> int:
    if blocks.dtype != torch.uint8 or blocks.dim() != 3 or K % 32 != 0 or blocks.shape[1:] != (K // 32, 18):
        raise ValueError("blocks must be uint8 [N, K/32, 18] with K a multiple of 32")
    if not blocks.is_contiguous():
        raise ValueError("blocks must be contiguous")
    return blocks.shape[0]


def dequantize_q4_0(blocks: torch.Tensor, K: int, out_dtype=torch.float32,
                    out: torch.Tensor | None = None) -> torch.Tensor:
    """Dense ``[N, K]`` weight of ``out_dtype`` from GGUF Q4_0 blocks (uint8 ``[N, K/32, 18]``)."""
    _need_cuda(blocks, out)
    N = _q4_0_shape(blocks, K)
    if out_dtype not in DTYPES:
        raise ValueError("unsupported output dtype")
    if out is None:
        out = torch.empty((N, K), dtype=out_dtype, device=blocks.device)
    _check(_load().w4_dequantize_q4_0(_ptr(blocks), N, K, DTYPES[out.dtype], _ptr(out), _stream()),
           "w4_dequantize_q4_0")
    return out


def q4_0_to_group32(blocks: torch.Tensor, K: int, out: tuple[torch.Tensor, torch.Tensor] | None = None):
    """GGUF Q4_0 blocks (uint8 ``[N, K/32, 18]``) re-laid out once as the packed group-32 format:
    returns ``(codes, scales)`` (uint8 ``[N, K/2]``, float32 ``[N, K/32]``; signed codes
    ``c - 8``, scales ``d`` widened to fp32) for ``linear`` / ``Linear`` / ``dequantize``, which
    then see exactly the blocks' dequantized weights."""
    _need_cuda(blocks)
    N = _q4_0_shape(blocks, K)
    if out is None:
        out = (torch.empty((N, K // 2), dtype=torch.uint8, device=blocks.device),
               torch.empty((N, K // 32), dtype=torch.float32, device=blocks.device))
    codes, scales = out
    _need_cuda(codes, scales)
    if not (codes.dtype == torch.uint8 and codes.is_contiguous() and codes.numel() == N * (K // 2)
            and scales.dtype == torch.float32 and scales.is_contiguous() and scales.numel() == N * (K // 32)):
        raise ValueError("out must be contiguous uint8 [N, K/2] codes and float32 [N, K/32] scales")
    _check(_load().w4_q4_0_to_group32(_ptr(blocks), N, K, _ptr(codes), _ptr(scales), _stream()),
           "w4_q4_0_to_group32")
    return codes, scales


def linear_q4_0(x: torch.Tensor, blocks: torch.Tensor, bias: torch.Tensor | None = None,
                out_dtype=torch.bfloat16, out: torch.Tensor | None = None) -> torch.Tensor:
    """``y = x . dequant(W)^T + bias`` for GGUF Q4_0 blocks; bf16 ``x [M, K]``, ``y [M, N]``."""
    _need_cuda(x, blocks, bias, out)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D bfloat16 tensor")
    M, K = x.shape
    N = _q4_0_shape(blocks, K)
    if bias is not None and (bias.dtype != torch.float32 or bias.numel() != N):
        raise ValueError("bias must be float32 [N]")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    if out.dtype not in (torch.bfloat16, torch.float32) or out.numel() != M * N or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 or float32 [M, N] tensor")
    _check(_load().w4_linear_q4_0(_ptr(x), M, _ptr(blocks), N, K, _ptr(bias), _ptr(out), DTYPES[out.dtype],
                                  _stream()), "w4_linear_q4_0")
    return out


_WS_BYTES = {}


def workspace_bytes(M: int, N: int, K: int) -> int:
    """Workspace the symmetric linear needs for these sizes (a function of the sizes only;
    cached per size triple)."""
    key = (M, N, K)
    v = _WS_BYTES.get(key)
    if v is None:
        v = int(_load().w4_linear_workspace_bytes(M, N, K))
        if len(_WS_BYTES) < 4096:
            _WS_BYTES[key] = v
    return v


def asym_workspace_bytes(M: int, N: int, K: int, n_groups: int) -> int:
    return int(_load().w4_linear_asym_workspace_bytes(M, N, K, n_groups))


def _workspace(M, N, K, device, workspace, need=None):
    if need is None:
        need = workspace_bytes(M, N, K)
    if need == 0:
        return None, 0
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


def linear(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, K: int | None = None,
           bias: torch.Tensor | None = None, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None) -> torch.Tensor:
    """``y = x . dequant(W)^T + bias`` for bf16 ``x [M, K]``; ``y [M, N]`` bf16 or fp32."""
    _need_cuda(x, codes, scales, bias, out, workspace)
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a 2-D bfloat16 tensor")
    M, Kx = x.shape
    K = Kx if K is None else K
    if K != Kx:
        raise ValueError("x width does not match K")
    N = codes.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    ws, wsb = _workspace(M, N, K, x.device, workspace)
    _check(_load().w4_linear(_ptr(x), M, _ptr(codes), _ptr(scales), N, K, _ptr(bias), _ptr(out),
                         DTYPES[out.dtype], _ptr(ws), wsb, _stream()), "w4_linear")
    return out


def linear_backward_x(dy: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, K: int,
                      out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Input gradient ``dx = dy . dequant(W)`` of :func:`linear`: bf16 ``dy [M, N]`` ->
    ``dx [M, K]`` (bf16 or fp32)."""
    _need_cuda(dy, codes, scales, out, workspace)
    if dy.dtype != torch.bfloat16 or dy.dim() != 2:
        raise ValueError("dy must be a 2-D bfloat16 tensor")
    M, N = dy.shape
    if codes.shape != (N, (K + 1) // 2) or scales.shape != (N, (K + 31) // 32):
        raise ValueError("codes / scales do not match dy and K")
    if out is None:
        out = torch.empty((M, K), dtype=out_dtype, device=dy.device)
    if out.dtype not in (torch.bfloat16, torch.float32) or out.numel() != M * K:
        raise ValueError("out must be a bf16 or float32 [M, K] tensor")
    need = int(_load().w4_linear_backward_x_workspace_bytes(M, N, K))
    ws, wsb = _workspace(M, N, K, dy.device, workspace, need=need)
    _check(_load().w4_linear_backward_x(_ptr(dy), M, _ptr(codes), _ptr(scales), N, K, _ptr(out), DTYPES[out.dtype],
                                        _ptr(ws), wsb, _stream()), "w4_linear_backward_x")
    return out


class Linear:
    """A prepared symmetric linear: ``Linear(codes, scales, bias)(x, out)`` computes what
    ``linear`` does, with the weight-side arguments checked and converted once (a layer
    called every decode step pays only the per-call part: x and out). The weights are
    referenced, not copied: keep them alive and unchanged while the object is used."""

    __slots__ = ("codes", "scales", "bias", "N", "K", "_codes_p", "_scales_p", "_bias_p", "_fn")

    def __init__(self, codes: torch.Tensor, scales: torch.Tensor, bias: torch.Tensor | None = None,
                 K: int | None = None):
        _need_cuda(codes, scales, bias)
        if codes.dtype != torch.uint8 or scales.dtype != torch.float32 or codes.dim() != 2 or scales.dim() != 2:
            raise ValueError("codes must be uint8 [N, ceil(K/2)] and scales float32 [N, ceil(K/32)]")
        N = codes.shape[0]
        K = 2 * codes.shape[1] if K is None else K
        if codes.shape[1] != (K + 1) // 2 or scales.shape != (N, (K + 31) // 32):
            raise ValueError("codes / scales do not match K")
        if bias is not None and (bias.dtype != torch.float32 or bias.numel() != N):
            raise ValueError("bias must be float32 [N]")
        if workspace_bytes(1, N, K) != 0:
            raise ValueError("this build's linear needs a workspace; use linear()")
        self.codes, self.scales, self.bias, self.N, self.K = codes, scales, bias, N, K
        self._codes_p, self._scales_p = codes.data_ptr(), scales.data_ptr()
        self._bias_p = None if bias is None else bias.data_ptr()
        self._fn = _load().w4_linear

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, out_dtype=torch.bfloat16) -> torch.Tensor:
        if not (x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 2 and x.shape[1] == self.K
                and x.is_contiguous()):
            raise ValueError("x must be a contiguous bfloat16 CUDA tensor [M, K]")
        M = x.shape[0]
        if out is None:
            out = torch.empty((M, self.N), dtype=out_dtype, device=x.device)
        elif not (out.is_cuda and out.is_contiguous() and out.dtype in (torch.bfloat16, torch.float32)
                  and out.numel() == M * self.N):
            raise ValueError("out must be a contiguous bf16 or fp32 CUDA tensor [M, N]")
        st = self._fn(x.data_ptr(), M, self._codes_p, self._scales_p, self.N, self.K, self._bias_p, out.data_ptr(),
                      0 if out.dtype == torch.bfloat16 else 2, None, 0, _stream())
        if st != 0:
            raise W4Error(st, "w4_linear")
        return out


def asym_prepare(codes: torch.Tensor, g_idx: torch.Tensor, K: int, n_groups: int):
    """Sort the act-order columns by group: returns ``(codes_sorted, perm)``."""
    _need_cuda(codes, g_idx)
    N = codes.shape[0]
    out = torch.empty_like(codes)
    perm = torch.empty(K, dtype=torch.int32, device=codes.device)
    _check(_load().w4_asym_prepare(_ptr(codes), _ptr(g_idx), N, K, n_groups, _ptr(out), _ptr(perm), _stream()),
           "w4_asym_prepare")
    return out, perm


def linear_asym_gidx(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                     g_idx: torch.Tensor, perm: torch.Tensor | None = None, bias: torch.Tensor | None = None,
                     out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Asymmetric act-order linear. ``g_idx`` may be float32 as Keras stores it; it is cast
    to int32 (exact below 2**24)."""
    if g_idx.dtype != torch.int32:
        g_idx = g_idx.to(torch.int32)
    _need_cuda(x, codes, scales, zeros, g_idx, perm, bias, out, workspace)
    M, K = x.shape
    N, G = scales.shape
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    need = asym_workspace_bytes(M, N, K, G) if perm is not None else 0
    ws, wsb = _workspace(M, N, K, x.device, workspace, need)
    _check(_load().w4_linear_asym_gidx(_ptr(x), M, _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(g_idx), _ptr(perm),
                                   N, K, G, _ptr(bias), _ptr(out), DTYPES[out.dtype], _ptr(ws), wsb,
                                   _stream()), "w4_linear_asym_gidx")
    return out


def linear_asym_gidx_noalloc(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                             g_idx: torch.Tensor, perm: torch.Tensor | None = None,
                             bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                             out_dtype=torch.bfloat16) -> torch.Tensor:
    """``linear_asym_gidx`` through the entry point that allocates no device memory (its
    scratch is a fixed 16 MiB array inside the library); pass ``out`` to allocate nothing
    on this side either."""
    if g_idx.dtype != torch.int32:
        raise ValueError("g_idx must be int32 here (the conversion would allocate)")
    _need_cuda(x, codes, scales, zeros, g_idx, perm, bias, out)
    M, K = x.shape
    N, G = scales.shape
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=x.device)
    _check(_load().w4_linear_asym_gidx_noalloc(_ptr(x), M, _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(g_idx),
                                           _ptr(perm), N, K, G, _ptr(bias), _ptr(out), DTYPES[out.dtype],
                                           _stream()), "w4_linear_asym_gidx_noalloc")
    return out


def validate(codes: torch.Tensor, scales: torch.Tensor, K: int, format_version: int = 2) -> str:
    """LoopQ content checks on the device; returns the status name ("OK" if valid)."""
    _need_cuda(codes, scales)
    return STATUS[_load().w4_validate(_ptr(codes), _ptr(scales), codes.shape[0], K, format_version, _stream())]


def validate_asym(codes, scales, zeros, g_idx, K: int) -> str:
    _need_cuda(codes, scales, zeros, g_idx)
    return STATUS[_load().w4_validate_asym(_ptr(codes), _ptr(scales), _ptr(zeros), _ptr(g_idx), codes.shape[0], K,
                                       scales.shape[1], _stream())]


def set_weight_prefetch(enable: bool) -> bool:
    """Decode launch policy: stream codes/scales before the previous kernel of the stream
    has finished (see w4_set_weight_prefetch in include/w4.h for the contract). Returns the
    previous setting."""
    return bool(_load().w4_set_weight_prefetch(1 if enable else 0))


def device_error() -> str:
    return STATUS[_load().w4_device_error()]


def last_linear_kernel() -> str:
    """Kernel family the calling thread's last linear call launched (``"none"`` before any)."""
    return _load().w4_last_linear_kernel().decode()


def selftest_wait_timeout(limit_ns: int) -> None:
    """Make one bounded device wait expire after ``limit_ns`` (diagnostic; see the header):
    the next ``device_error()`` reports ``"TIMEOUT"``."""
    _check(_load().w4_selftest_wait_timeout(int(limit_ns), _stream()), "selftest_wait_timeout")
