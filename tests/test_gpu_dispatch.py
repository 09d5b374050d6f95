"""Which kernel serves which linear call: every kernel behind w4_linear /
w4_linear_asym_gidx is reached by at least one case here, asserted through
w4_last_linear_kernel(), and each case's output is checked against the oracle at the linear
tolerance. The cases name the property that routes them (M, K alignment, array alignment,
scale-group counts, act-order preparation, workspace)."""

import numpy as np
import pytest
import torch

import oracle as O
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from weight_only_int4_04_b200 import build
    build.build()
    import weight_only_int4_04_b200 as w
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return w


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _x(bits):
    return _dev(bits.view(np.int16)).view(torch.bfloat16)


SYM_CASES = [
    # (M, N, K, x_offset_bytes, expected kernel, why)
    (1, 300, 4096, 0, "gemv_tma", "M = 1, K a multiple of 128, aligned arrays"),
    (1, 300, 2176, 0, "gemv_tma", "M = 1, K a multiple of 128 but not of 1024 (one 2-D box per k-tile)"),
    (8, 300, 2048, 0, "gemv_tma", "2 <= M <= 8: one n-tile"),
    (16, 300, 2048, 0, "gemv_tma", "9 <= M <= 16: two n-tiles"),
    (1, 300, 1056, 0, "gemv_rows", "M = 1, K % 128 != 0 (no TMA boxes), packed rows a multiple of 16 bytes"),
    (1, 300, 2048, 8, "gemv_rows", "M = 1, x 8 bytes past a 16-byte boundary"),
    (5, 300, 1023, 0, "gemv_mma", "2 <= M <= 16, K % 128 != 0, scale groups a multiple of 4"),
    (3, 300, 1056, 0, "gemv", "M <= 4, 33 scale groups (not a multiple of 4)"),
    (1, 64, 28704, 0, "gemv", "M = 1, K past the register-streaming kernel's 28672"),
    (17, 300, 4096, 0, "gemm_tc", "M >= 17, aligned"),
    (64, 300, 4096, 0, "gemm_tc", "the 64-row activation tile"),
    (300, 300, 2048, 0, "gemm_tc", "the 256-row activation tile, ragged"),
    (5, 300, 1001, 0, "linear_generic", "odd K: packed rows not a multiple of 16 bytes"),
    (20, 300, 1000, 0, "linear_generic", "M >= 17 with packed rows of 500 bytes"),
]


@pytest.mark.parametrize("case", SYM_CASES, ids=[f"{c[4]}-M{c[0]}-K{c[2]}-off{c[3]}" for c in SYM_CASES])
def test_symmetric_dispatch(w4, case):
    M, N, K, off, expect, _why = case
    c = workloads.linear_case(M * 7 + K + off, M, N, K, outliers=True)
    q, s = O.quantize_rtn(c["W"])
    codes = O.pack_nibbles(q)
    x = _x(c["x_bits"])
    if off:
        buf = torch.zeros(M * K + off // 2 + 8, dtype=torch.bfloat16, device="cuda")
        xv = buf[off // 2: off // 2 + M * K].view(M, K)
        xv.copy_(x)
        assert xv.data_ptr() % 16 == off
        x = xv
    y = w4.linear(x, _dev(codes), _dev(s), K, bias=_dev(c["bias"]), out_dtype=torch.float32)
    assert w4.last_linear_kernel() == expect
    yr, bound = O.linear(c["x"], codes, s, K, c["bias"])
    ok, worst = O.check_linear(y.cpu().numpy().astype(np.float64), yr, bound)
    assert ok, worst


ASYM_CASES = [
    # (M, K, group, prepared, expected kernel)
    (1, 4096, 128, True, "gemv_tma"),            # one row: gathered inside the GEMV
    (4, 4096, 128, True, "gather_x+gemv_tma"),   # several rows: one gather kernel into the workspace
    (32, 4096, 128, True, "gather_x+gemm_tc"),   # M >= 17: gathered, then the tcgen05 GEMM
    (4, 4096, 128, False, "linear_generic"),     # unprepared codes (no column sort)
    (40, 1024, 96, True, "linear_generic"),      # M >= 17 with 11 groups (not a multiple of 16)
]


@pytest.mark.parametrize("case", ASYM_CASES, ids=[f"{c[4]}-M{c[0]}-g{c[2]}-{'prep' if c[3] else 'raw'}"
                                                  for c in ASYM_CASES])
def test_asym_dispatch(w4, case):
    M, K, group, prepared, expect = case
    N = 256
    a = workloads.asym_case(M=M, N=N, K=K, group=group, seed=M + K + group)
    u, s, z = O.quantize_asym_minmax(a["W"], a["g_idx"], a["n_groups"])
    codes = O.pack_nibbles(u)
    gi = _dev(a["g_idx"])
    if prepared:
        dc, perm = w4.asym_prepare(_dev(codes), gi, K, a["n_groups"])
    else:
        dc, perm = _dev(codes), None
    y = w4.linear_asym_gidx(_x(a["x_bits"]), dc, _dev(s), _dev(z), gi, perm=perm, bias=_dev(a["bias"]),
                            out_dtype=torch.float32)
    assert w4.last_linear_kernel() == expect
    yr, bound = O.linear_asym_gidx(a["x"], codes, s, z, a["g_idx"], K, a["bias"])
    ok, worst = O.check_linear(y.cpu().numpy().astype(np.float64), yr, bound)
    assert ok, worst
