"""C-ABI checks that need no GPU: the library builds for sm_100a, loads, exports every
entry point include/w4.h declares, and its host-side argument checks return the
documented status codes before anything is enqueued."""

import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "w4.h")


@pytest.fixture(scope="module")
def w4():
    from weight_only_int4_04_b200 import build
    build.build()
    import weight_only_int4_04_b200 as w
    return w


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(w4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("w4_quantize_rtn", "w4_dequantize", "w4_linear", "w4_linear_asym_gidx"):
        assert required in names


def test_library_exports_every_declared_symbol(w4):
    lib = ctypes.CDLL(w4.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(w4.EXPORTS) | set(declared_functions())
    assert w4.lib.w4_version() >= 100


def test_status_strings(w4):
    for code in w4.STATUS:
        assert w4.lib.w4_status_string(code)
    assert b"finite" in w4.lib.w4_status_string(5)


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails its host check


def test_null_pointers_rejected(w4):
    L = w4.lib
    assert L.w4_quantize_rtn(None, 4, 32, FAKE, FAKE, None, None) == 1
    assert L.w4_dequantize(FAKE, None, 4, 32, 2, 0, FAKE, None) == 1
    assert L.w4_linear(FAKE, 1, FAKE, FAKE, 4, 32, None, None, 0, None, 0, None) == 1
    assert L.w4_linear_asym_gidx(FAKE, 1, FAKE, FAKE, None, FAKE, None, 4, 32, 1, None, FAKE, 0, None, 0,
                                 None) == 1
    assert L.w4_validate(None, FAKE, 4, 32, 2, None) == 1
    assert L.w4_asym_prepare(FAKE, FAKE, 4, 32, 1, None, FAKE, None) == 1


@pytest.mark.parametrize("N,K", [(0, 32), (4, 0), (-1, 5), (4, (1 << 24) + 1), (1 << 31, 4)])
def test_bad_sizes_rejected(w4, N, K):
    L = w4.lib
    assert L.w4_quantize_rtn(FAKE, N, K, FAKE, FAKE, None, None) == 2
    assert L.w4_dequantize(FAKE, FAKE, N, K, 2, 0, FAKE, None) == 2
    assert L.w4_linear(FAKE, 1, FAKE, FAKE, N, K, None, FAKE, 0, None, 0, None) == 2
    assert L.w4_validate(FAKE, FAKE, N, K, 2, None) == 2


def test_bad_m_and_groups_rejected(w4):
    L = w4.lib
    assert L.w4_linear(FAKE, 0, FAKE, FAKE, 4, 32, None, FAKE, 0, None, 0, None) == 2
    assert L.w4_linear_asym_gidx(FAKE, 1, FAKE, FAKE, FAKE, FAKE, None, 4, 32, 0, None, FAKE, 0, None, 0,
                                 None) == 2
    assert L.w4_linear_asym_gidx(FAKE, 1, FAKE, FAKE, FAKE, FAKE, None, 4, 32, 33, None, FAKE, 0, None, 0,
                                 None) == 2


def test_dtype_and_version_rejected(w4):
    L = w4.lib
    assert L.w4_dequantize(FAKE, FAKE, 4, 32, 2, 7, FAKE, None) == 3
    assert L.w4_linear(FAKE, 1, FAKE, FAKE, 4, 32, None, FAKE, 1, None, 0, None) == 3  # f16 y not offered
    assert L.w4_linear(FAKE, 1, FAKE, FAKE, 4, 32, None, FAKE, 3, None, 0, None) == 3
    assert L.w4_dequantize(FAKE, FAKE, 4, 32, 3, 0, FAKE, None) == 8
    assert L.w4_dequantize(FAKE, FAKE, 4, 32, 0, 0, FAKE, None) == 8
    assert L.w4_validate(FAKE, FAKE, 4, 32, 5, None) == 8


def test_binding_refuses_cpu_tensors(w4):
    import torch
    with pytest.raises(ValueError):
        w4.quantize_rtn(torch.zeros(4, 32))
    with pytest.raises(ValueError):
        w4.linear(torch.zeros(1, 32, dtype=torch.bfloat16), torch.zeros(4, 16, dtype=torch.uint8),
                  torch.ones(4, 1))


def test_workspace_query(w4):
    assert w4.workspace_bytes(1, 4096, 4096) >= 0


def test_prepared_linear_requires_cuda_tensors():
    """w4.Linear refuses host tensors (no CPU fallback), before touching the library."""
    import torch

    import weight_only_int4_04_b200 as w4
    with pytest.raises(ValueError):
        w4.Linear(torch.zeros((4, 8), dtype=torch.uint8), torch.ones((4, 1), dtype=torch.float32))


def test_q4_0_host_checks(w4):
    L = w4.lib
    FAKE = ctypes.c_void_p(0x1000)
    # NULL pointers, K not a multiple of 32, bad sizes, bad dtypes: rejected before any launch
    assert L.w4_linear_q4_0(None, 1, FAKE, 4, 64, None, FAKE, 0, None) == 1
    assert L.w4_linear_q4_0(FAKE, 1, None, 4, 64, None, FAKE, 0, None) == 1
    assert L.w4_dequantize_q4_0(None, 4, 64, 2, FAKE, None) == 1
    assert L.w4_linear_q4_0(FAKE, 1, FAKE, 4, 48, None, FAKE, 0, None) == 2
    assert L.w4_linear_q4_0(FAKE, 0, FAKE, 4, 64, None, FAKE, 0, None) == 2
    assert L.w4_linear_q4_0(FAKE, 1, FAKE, 0, 64, None, FAKE, 0, None) == 2
    assert L.w4_dequantize_q4_0(FAKE, 4, 40, 2, FAKE, None) == 2
    assert L.w4_linear_q4_0(FAKE, 1, FAKE, 4, 64, None, FAKE, 1, None) == 3  # f16 y not offered
    assert L.w4_dequantize_q4_0(FAKE, 4, 64, 9, FAKE, None) == 3


def test_q4_0_binding_refuses_cpu_and_bad_shapes(w4):
    import torch
    blocks = torch.zeros((4, 2, 18), dtype=torch.uint8)
    x = torch.zeros((1, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        w4.linear_q4_0(x, blocks)
    with pytest.raises(ValueError):
        w4.dequantize_q4_0(blocks, 64)


def test_backward_host_checks(w4):
    L = w4.lib
    FAKE = ctypes.c_void_p(0x1000)
    assert L.w4_linear_backward_x(None, 1, FAKE, FAKE, 4, 64, FAKE, 0, None, 0, None) == 1
    assert L.w4_linear_backward_x(FAKE, 0, FAKE, FAKE, 4, 64, FAKE, 0, None, 0, None) == 2
    assert L.w4_linear_backward_x(FAKE, 1, FAKE, FAKE, 4, 64, FAKE, 3, None, 0, None) == 3
    need = L.w4_linear_backward_x_workspace_bytes(1, 14336, 4096)
    assert need > 0 and L.w4_linear_backward_x_workspace_bytes(1, 14336, 4096) == need
    assert L.w4_linear_backward_x(FAKE, 1, FAKE, FAKE, 14336, 4096, FAKE, 0, None, 0, None) == 12
    assert L.w4_linear_backward_x_workspace_bytes(1, 8, 37) == 0  # plain kernel: none


def test_channel_host_checks(w4):
    L = w4.lib
    FAKE = ctypes.c_void_p(0x1000)
    assert L.w4_quantize_rtn_channel(None, 4, 64, FAKE, FAKE, None, None) == 1
    assert L.w4_quantize_rtn_channel(FAKE, 0, 64, FAKE, FAKE, None, None) == 2
    assert L.w4_expand_channel_scales(FAKE, 4, 0, FAKE, None) == 2
    assert L.w4_expand_channel_scales(None, 4, 64, FAKE, None) == 1


def test_lora_host_checks(w4):
    L = w4.lib
    FAKE = ctypes.c_void_p(0x1000)
    c = ctypes.c_float(1.0)
    assert L.w4_lora_merge(None, FAKE, 4, 64, FAKE, FAKE, 2, c, FAKE, FAKE, None, None) == 1
    assert L.w4_lora_merge(FAKE, FAKE, 4, 64, None, FAKE, 2, c, FAKE, FAKE, None, None) == 1
    assert L.w4_lora_merge(FAKE, FAKE, 4, 64, FAKE, FAKE, -1, c, FAKE, FAKE, None, None) == 2
    assert L.w4_lora_merge(FAKE, FAKE, 0, 64, FAKE, FAKE, 2, c, FAKE, FAKE, None, None) == 2


def test_q4_0_to_group32_host_checks(w4):
    L = w4.lib
    FAKE = ctypes.c_void_p(0x1000)
    assert L.w4_q4_0_to_group32(None, 4, 64, FAKE, FAKE, None) == 1
    assert L.w4_q4_0_to_group32(FAKE, 4, 64, None, FAKE, None) == 1
    assert L.w4_q4_0_to_group32(FAKE, 4, 64, FAKE, None, None) == 1
    assert L.w4_q4_0_to_group32(FAKE, 4, 48, FAKE, FAKE, None) == 2  # K not a multiple of 32
    assert L.w4_q4_0_to_group32(FAKE, 0, 64, FAKE, FAKE, None) == 2
    import torch
    with pytest.raises(ValueError):  # CPU tensors: no fallback
        w4.q4_0_to_group32(torch.zeros((4, 2, 18), dtype=torch.uint8), 64)


def test_new_bindings_validate_arguments(w4):
    import torch
    f32 = torch.zeros((4, 64), dtype=torch.float32)
    with pytest.raises(ValueError):  # CPU tensors: no fallback
        w4.quantize_rtn_channel(f32)
    with pytest.raises(ValueError):
        w4.expand_channel_scales(torch.zeros(4), 64)
    with pytest.raises(ValueError):
        w4.linear_backward_x(torch.zeros((1, 4), dtype=torch.bfloat16), torch.zeros((4, 32), dtype=torch.uint8),
                             torch.zeros((4, 2), dtype=torch.float32), 64)
    with pytest.raises(ValueError):
        w4.lora_merge(torch.zeros((4, 32), dtype=torch.uint8), torch.zeros((4, 2)), 64, torch.zeros((4, 2)),
                      torch.zeros((2, 64)), 1.0)


def test_wait_selftest_host_checks(w4):
    """The wait self-test refuses a zero limit and one above the library's own 1 s limit
    before anything is enqueued."""
    assert w4.STATUS[w4.lib.w4_selftest_wait_timeout(0, None)] == "SHAPE"
    assert w4.STATUS[w4.lib.w4_selftest_wait_timeout(10**9 + 1, None)] == "SHAPE"


def test_linear_channel_host_checks(w4):
    L = w4.lib
    assert w4.STATUS[L.w4_linear_channel(None, 1, FAKE, FAKE, 4, 128, None, FAKE, 0, None, 0, None)] == "NULL"
    assert w4.STATUS[L.w4_linear_channel(FAKE, 0, FAKE, FAKE, 4, 128, None, FAKE, 0, None, 0, None)] == "SHAPE"
    assert w4.STATUS[L.w4_linear_channel(FAKE, 1, FAKE, FAKE, 4, 128, None, FAKE, 3, None, 0, None)] == "DTYPE"
    assert int(L.w4_linear_channel_workspace_bytes(1, 64, 4096)) == 0
    assert int(L.w4_linear_channel_workspace_bytes(17, 64, 4096)) == 64 * 128 * 4
