"""GPU parity of w4_linear_backward_x (through the C ABI) against the oracle's
linear_backward_x on the same seeded weights and upstream gradients:
|dx - dx_ref| <= 4e-3 * sum_n |dy w| + 1e-6 per element. Shapes span the streaming kernel
(K a multiple of 8: one to several row splits, ragged column tiles, 1 to 33 upstream rows)
and the plain kernel (other K)."""

import numpy as np
import pytest
import torch

import oracle.w4_oracle as O
import workloads

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


def case(M, N, K, seed):
    c = workloads.linear_case(seed, 1, N, K, bias=False)
    q, s = O.quantize_rtn(c["W"])
    codes = O.pack_nibbles(q)
    dy_bits, dy = workloads.draw_x(np.random.default_rng([7, seed]), M, N)
    return codes, s, dy_bits, dy


def check(dx, dxr, bound, ctx):
    err = np.abs(dx - dxr)
    lim = 4e-3 * bound + 1e-6
    assert np.all(err <= lim), (ctx, float((err / lim).max()))


CASES = [(1, 1, 8), (1, 64, 256), (1, 300, 4096), (1, 4100, 1000), (2, 129, 520), (3, 700, 2048), (8, 96, 264),
         (16, 1024, 4096), (33, 200, 512), (1, 17, 37), (4, 33, 99), (2, 5, 1)]


@pytest.mark.parametrize("MNK", CASES, ids=[f"M{m}_N{n}_K{k}" for m, n, k in CASES])
def test_backward_x(w4, MNK):
    M, N, K = MNK
    codes, s, dy_bits, dy = case(M, N, K, M * 131 + N * 7 + K)
    dxr, bound = O.linear_backward_x(dy, codes, s, K)
    for dt in (torch.float32, torch.bfloat16):
        dx = w4.linear_backward_x(bf16_dev(dy_bits), dev(codes), dev(s), K, out_dtype=dt)
        check(dx.float().cpu().numpy().astype(np.float64), dxr, bound, (M, N, K, str(dt)))


def test_backward_x_full_size_and_deterministic(w4):
    N, K = workloads.BATCHED_SHAPE
    codes, s, dy_bits, dy = case(1, N, K, 3)
    dxr, bound = O.linear_backward_x(dy, codes, s, K)
    dc, ds, ddy = dev(codes), dev(s), bf16_dev(dy_bits)
    a = w4.linear_backward_x(ddy, dc, ds, K, out_dtype=torch.float32)
    b = w4.linear_backward_x(ddy, dc, ds, K, out_dtype=torch.float32)
    check(a.cpu().numpy().astype(np.float64), dxr, bound, "full")
    assert torch.equal(a, b)  # fixed-order sums: bitwise repeatable


def test_backward_x_one_hot_exact(w4):
    N, K = 48, 512
    codes, s, _, _ = case(1, N, K, 11)
    w = O.dequantize(codes, s, K, "f32")
    dc, ds = dev(codes), dev(s)
    for n in (0, 7, 47):
        dy = np.zeros((1, N), np.float32)
        dy[0, n] = 1.0
        dx = w4.linear_backward_x(bf16_dev(O.f32_to_bf16_bits(dy)), dc, ds, K, out_dtype=torch.float32)
        assert np.array_equal(dx.cpu().numpy()[0], w[n]), n


def test_backward_x_is_adjoint_of_linear(w4):
    """<y, dy> = <x, dx> with both sides from the GPU (within the two tolerances)."""
    M, N, K = 4, 384, 1024
    c = workloads.linear_case(21, M, N, K, bias=False)
    q, s = O.quantize_rtn(c["W"])
    codes = O.pack_nibbles(q)
    dy_bits, dy = workloads.draw_x(np.random.default_rng(5), M, N)
    y = w4.linear(bf16_dev(c["x_bits"]), dev(codes), dev(s), K, out_dtype=torch.float32).cpu().numpy()
    dx = w4.linear_backward_x(bf16_dev(dy_bits), dev(codes), dev(s), K, out_dtype=torch.float32).cpu().numpy()
    lhs = float((y.astype(np.float64) * dy).sum())
    rhs = float((dx.astype(np.float64) * c["x"]).sum())
    w = O.dequantize(codes, s, K, "f32").astype(np.float64)
    # sum over (m, n, k) of |x w dy|: each side is within 4e-3 of it
    scale = float(((np.abs(c["x"].astype(np.float64)) @ np.abs(w).T) * np.abs(dy)).sum())
    assert abs(lhs - rhs) <= 8e-3 * scale


# the tensor-core kernel (2 <= M, K a multiple of 128, N a multiple of 8): ragged 32-row steps,
# several 16-row token tiles, row splits, the full-size shape
MMA_CASES = [(2, 64, 128), (5, 1000, 384), (16, 14336, 4096), (64, 2048, 1024), (17, 8, 256), (40, 3000, 640)]


@pytest.mark.parametrize("MNK", MMA_CASES, ids=[f"M{m}_N{n}_K{k}" for m, n, k in MMA_CASES])
def test_backward_x_tensor_core(w4, MNK):
    M, N, K = MNK
    codes, s, dy_bits, dy = case(M, N, K, M * 17 + N + K)
    dxr, bound = O.linear_backward_x(dy, codes, s, K)
    ddy, dc, ds = bf16_dev(dy_bits), dev(codes), dev(s)
    for dt in (torch.float32, torch.bfloat16):
        dx = w4.linear_backward_x(ddy, dc, ds, K, out_dtype=dt)
        check(dx.float().cpu().numpy().astype(np.float64), dxr, bound, (M, N, K, str(dt)))
    a = w4.linear_backward_x(ddy, dc, ds, K, out_dtype=torch.float32)
    b = w4.linear_backward_x(ddy, dc, ds, K, out_dtype=torch.float32)
    assert torch.equal(a, b)  # fixed-order split sums: bitwise repeatable


def test_backward_x_tensor_core_one_hot(w4):
    """One-hot upstream rows pick one weight row. The tensor-core kernel carries each weight
    as a pair of bf16 values whose sum is within 2^-16 of the fp32 dequantized weight, so dx
    must match that row to 2^-15 relative -- far inside the linear tolerance, and far from
    what a single bf16 weight (2^-8) would give."""
    M, N, K = 4, 96, 512
    codes, s, _, _ = case(M, N, K, 12)
    w = O.dequantize(codes, s, K, "f32").astype(np.float64)
    rows = [0, 31, 32, 95]
    dy = np.zeros((M, N), np.float32)
    for m, n in enumerate(rows):
        dy[m, n] = 1.0
    dx = w4.linear_backward_x(bf16_dev(O.f32_to_bf16_bits(dy)), dev(codes), dev(s), K, out_dtype=torch.float32)
    got = dx.cpu().numpy().astype(np.float64)
    for m, n in enumerate(rows):
        assert np.all(np.abs(got[m] - w[n]) <= 2.0**-15 * np.abs(w[n])), (m, n)
