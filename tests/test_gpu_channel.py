"""GPU parity of the per-channel entry points (w4_quantize_rtn_channel,
w4_expand_channel_scales; C ABI) against the per-channel oracle: codes and scales
bit-identical, expanded scales exact, and the group-32 kernels (linear, dequant, input
gradient) serving the expanded weight within the linear's tolerance of the oracle."""

import numpy as np
import pytest
import torch

import oracle.w4_oracle as O
import workloads
from conftest import read_golden

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from weight_only_int4_04_b200 import build
    build.build()
    import weight_only_int4_04_b200 as w
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return w


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_dev(bits):
    return dev(bits.view(np.int16)).view(torch.bfloat16)


@pytest.mark.parametrize("NK", [(1, 1), (3, 7), (37, 333), (64, 4096), (5, 100001), (300, 1000)])
def test_channel_quantize_bit_exact(w4, NK):
    N, K = NK
    c = workloads.linear_case(N * 3 + K, 1, N, K, outliers=True, bias=False)
    W = c["W"].copy()
    if N > 2:
        W[1] = 0.0  # an all-zero row: floor scale, codes 0
    codes, scales = w4.quantize_rtn_channel(dev(W))
    q, s = O.quantize_rtn_channel(W)
    assert np.array_equal(codes.cpu().numpy(), O.pack_nibbles(q)), NK
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), s.view(np.uint32)), NK
    ex = w4.expand_channel_scales(scales, K)
    assert np.array_equal(ex.cpu().numpy(), O.expand_channel_scales(s, K))


def test_channel_worked_example_on_device(w4):
    g = read_golden("channel_worked_example.txt")
    W = np.stack([[float(v) for v in g[k]] for k in ("W0", "W1", "W2")]).astype(np.float32)
    codes, scales = w4.quantize_rtn_channel(dev(W))
    q = np.stack([[int(float(v)) for v in g[k]] for k in ("q0", "q1", "q2")]).astype(np.int8)
    assert np.array_equal(codes.cpu().numpy(), O.pack_nibbles(q))
    assert np.array_equal(scales.cpu().numpy().astype(np.float64), np.array([float(v) for v in g["scales"]]))


def test_channel_nonfinite_rejected(w4):
    W = np.ones((4, 64), np.float32)
    W[2, 17] = np.nan
    with pytest.raises(Exception):
        w4.quantize_rtn_channel(dev(W))


@pytest.mark.parametrize("MNK", [(1, 4096, 4096), (16, 1000, 2048), (64, 512, 1024), (3, 33, 96)])
def test_channel_linear_and_gradient(w4, MNK):
    M, N, K = MNK
    c = workloads.linear_case(M + N + K, M, N, K)
    codes, scales = w4.quantize_rtn_channel(dev(c["W"]))
    ex = w4.expand_channel_scales(scales, K)
    q, s = O.quantize_rtn_channel(c["W"])
    rc, rs = O.pack_nibbles(q), O.expand_channel_scales(s, K)
    y = w4.linear(bf16_dev(c["x_bits"]), codes, ex, K, bias=dev(c["bias"]), out_dtype=torch.float32)
    yr, bound = O.linear(c["x"], rc, rs, K, c["bias"])
    ok, worst = O.check_linear(y.cpu().numpy(), yr, bound)
    assert ok, (MNK, worst)
    deq = w4.dequantize(codes, ex, K, torch.float32)
    assert np.array_equal(deq.cpu().numpy(), O.dequantize(rc, rs, K, "f32"))
    dy_bits, dy = workloads.draw_x(np.random.default_rng(M), M, N)
    dx = w4.linear_backward_x(bf16_dev(dy_bits), codes, ex, K, out_dtype=torch.float32)
    dxr, dbound = O.linear_backward_x(dy, rc, rs, K)
    ok, worst = O.check_linear(dx.cpu().numpy(), dxr, dbound)
    assert ok, (MNK, "dx", worst)


# ---------------------------------------------------------------------------
# w4_linear_channel: one scale per row read by the decode kernel (M <= 16), or expanded into
# the workspace for the group-32 kernels (other shapes)
# ---------------------------------------------------------------------------

CHANNEL_LINEAR = [
    # (M, N, K, kernel expected)
    (1, 300, 4096, "gemv_tma_channel"),    # whole-stage 3-D boxes of codes
    (1, 4100, 2176, "gemv_tma_channel"),   # K % 1024 != 0: 2-D boxes per k-tile, ragged rows
    (1, 64, 14336, "gemv_tma_channel"),    # long rows: several stages per row block
    (5, 300, 4096, "gemv_tma_channel"),    # one n-tile of activation rows
    (16, 333, 2048, "gemv_tma_channel"),   # two n-tiles
    (17, 300, 4096, "gemm_tc"),            # expanded scales, tensor-core GEMM
    (3, 300, 1056, "gemv"),                # K % 128 != 0: expanded scales, CUDA-core GEMV
    (1, 257, 1001, "linear_generic"),      # odd K
]


@pytest.mark.parametrize("case", CHANNEL_LINEAR, ids=[f"M{c[0]}-N{c[1]}-K{c[2]}" for c in CHANNEL_LINEAR])
def test_linear_channel_matches_oracle(w4, case):
    M, N, K, expect = case
    c = workloads.linear_case(M * 5 + N + K, M, N, K, outliers=True)
    q, s = O.quantize_rtn_channel(c["W"])
    codes = O.pack_nibbles(q)
    y = w4.linear_channel(bf16_dev(c["x_bits"]), dev(codes), dev(s), K, bias=dev(c["bias"]),
                          out_dtype=torch.float32)
    assert w4.last_linear_kernel() == expect
    yr, bound = O.linear(c["x"], codes, O.expand_channel_scales(s, K), K, c["bias"])
    ok, worst = O.check_linear(y.cpu().numpy().astype(np.float64), yr, bound)
    assert ok, worst
    yb = w4.linear_channel(bf16_dev(c["x_bits"]), dev(codes), dev(s), K, bias=dev(c["bias"]))
    ok, worst = O.check_linear(yb.float().cpu().numpy().astype(np.float64), yr, bound)
    assert ok, worst


def test_linear_channel_one_hot_closed_form(w4):
    """x = e_k picks column k: y = q[:, k] * s + b, computed exactly by the decode kernel
    (one nonzero product per row, one scale multiply, one bias add, all in fp32)."""
    N, K = 300, 4096
    c = workloads.linear_case(4242, 1, N, K)
    q, s = O.quantize_rtn_channel(c["W"])
    codes = O.pack_nibbles(q)
    for k in (0, 1, 4095, 1234):
        xb = np.zeros((1, K), np.uint16)
        xb[0, k] = 0x3F80  # 1.0
        y = w4.linear_channel(bf16_dev(xb), dev(codes), dev(s), K, bias=dev(c["bias"]), out_dtype=torch.float32)
        assert w4.last_linear_kernel() == "gemv_tma_channel"
        want = (q[:, k].astype(np.float32) * s).astype(np.float32) + c["bias"]
        assert np.array_equal(y.cpu().numpy()[0], want.astype(np.float32))


def test_linear_channel_requires_workspace_off_the_decode_path(w4):
    import ctypes
    M, N, K = 20, 64, 1024
    c = workloads.linear_case(7, M, N, K)
    q, s = O.quantize_rtn_channel(c["W"])
    x, cd, sd = bf16_dev(c["x_bits"]), dev(O.pack_nibbles(q)), dev(s)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    need = int(w4.lib.w4_linear_channel_workspace_bytes(M, N, K))
    assert need >= N * (K // 32) * 4
    st = w4.lib.w4_linear_channel(w4._ptr(x), M, w4._ptr(cd), w4._ptr(sd), N, K, None, w4._ptr(y), 0, None, 0,
                                  w4._stream())
    assert w4.STATUS[st] == "WORKSPACE"
    assert int(w4.lib.w4_linear_channel_workspace_bytes(1, N, K)) == 0
