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
