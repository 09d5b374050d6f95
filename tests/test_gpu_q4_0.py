"""GPU parity of the GGUF Q4_0 entry points (w4_dequantize_q4_0, w4_linear_q4_0, called
through the C ABI) against the Q4_0 oracle on the same seeded blocks: dequantized weights
bit-identical in every output dtype; linear outputs within |y - y_ref| <= 4e-3 * sum_k |x w|
+ 1e-6 per element. Shapes span the TMA decode kernel (M = 1, K a multiple of 256: several
row blocks, ragged last row block, rows of 1 to 112 k-tiles, the three decode projections at
full size) and the plain kernel (other K, M > 1)."""

import numpy as np
import pytest
import torch

import oracle.q4_0 as Q
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


def x_dev(bits):
    return dev(bits.view(np.int16)).view(torch.bfloat16)


def special_blocks(N, K):
    """Blocks whose scales take the binary16 edge values (subnormal, largest, signed zero,
    negative) next to random ones."""
    b = workloads.q4_0_case(N * 7 + K, 1, N, K)["blocks"].copy()
    specials = [0x0001, 0x03FF, 0x0400, 0x7BFF, 0xFBFF, 0x8000, 0x0000, 0xC000, 0x3C00]
    flat = b.reshape(-1, 18)
    for i, bits in enumerate(specials[: flat.shape[0]]):
        flat[i * 3 % flat.shape[0], 0] = bits & 0xFF
        flat[i * 3 % flat.shape[0], 1] = bits >> 8
    return b


@pytest.mark.parametrize("NK", [(1, 32), (3, 96), (17, 256), (64, 1056), (129, 4096)])
def test_q4_0_dequant_bit_exact(w4, NK):
    N, K = NK
    blocks = special_blocks(N, K)
    db = dev(blocks)
    for dt, name in ((torch.float32, "f32"), (torch.float64, "f64"), (torch.bfloat16, "bf16"),
                     (torch.float16, "f16")):
        out = w4.dequantize_q4_0(db, K, dt).cpu()
        exp = Q.dequantize(blocks, K, name)
        if name == "bf16":
            got = out.view(torch.int16).numpy().view(np.uint16)
        elif name == "f16":
            got = out.view(torch.int16).numpy().view(np.uint16)
            exp = exp.view(np.uint16)
        else:
            got = out.numpy()
        assert np.array_equal(got.view(np.uint8), np.ascontiguousarray(exp).view(np.uint8)), (N, K, name)


def check(y, yr, bound, ctx):
    err = np.abs(y - yr)
    lim = 4e-3 * bound + 1e-6
    assert np.all(err <= lim), (ctx, float((err / lim).max()))


LINEAR_CASES = [
    # TMA decode kernel (M = 1, K % 256 == 0): one row, ragged row blocks, long rows
    (1, 1, 256), (1, 16, 256), (1, 17, 512), (1, 33, 2048), (1, 300, 4096), (1, 593, 1024),
    (1, 4100, 4096), (1, 7, 28672), (1, 2049, 3072), (1, 64, 14336),
    # plain kernel: K not a multiple of 256, several activation rows
    (1, 5, 96), (1, 64, 1056), (2, 33, 256), (5, 17, 4096), (16, 100, 1024), (9, 3, 32),
]


@pytest.mark.parametrize("case", LINEAR_CASES, ids=[f"M{m}_N{n}_K{k}" for m, n, k in LINEAR_CASES])
def test_q4_0_linear(w4, case):
    M, N, K = case
    c = workloads.q4_0_case(M * 1000003 + N * 101 + K, M, N, K)
    yr, bound = Q.linear(c["x"], c["blocks"], K, c["bias"])
    for dt in (torch.float32, torch.bfloat16):
        y = w4.linear_q4_0(x_dev(c["x_bits"]), dev(c["blocks"]), bias=dev(c["bias"]), out_dtype=dt)
        check(y.float().cpu().numpy().astype(np.float64), yr, bound, (M, N, K, str(dt)))
    y = w4.linear_q4_0(x_dev(c["x_bits"]), dev(c["blocks"]), out_dtype=torch.float32)
    yr0, _ = Q.linear(c["x"], c["blocks"], K, None)
    check(y.cpu().numpy().astype(np.float64), yr0, bound, (M, N, K, "no bias"))


@pytest.mark.parametrize("NK", workloads.Q4_0_SHAPES)
def test_q4_0_decode_full_size(w4, NK):
    N, K = NK
    c = workloads.q4_0_case(N + K, 1, N, K, bias=False)
    yr, bound = Q.linear(c["x"], c["blocks"], K)
    y = w4.linear_q4_0(x_dev(c["x_bits"]), dev(c["blocks"]), out_dtype=torch.float32)
    check(y.cpu().numpy().astype(np.float64), yr, bound, (N, K))


def test_q4_0_one_hot_exact(w4):
    N, K = 40, 512
    c = workloads.q4_0_case(77, 1, N, K)
    w = Q.dequantize(c["blocks"], K, "f32")
    db = dev(c["blocks"])
    for k in (0, 15, 16, 31, 32, 300, 511):
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        y = w4.linear_q4_0(x_dev(O.f32_to_bf16_bits(x)), db, bias=dev(c["bias"]), out_dtype=torch.float32)
        assert np.array_equal(y.cpu().numpy()[0], (w[:, k] + c["bias"]).astype(np.float32)), k


def test_q4_0_prefetch_policy_and_chain(w4):
    """Back-to-back decode calls with weight prefetch on and off, each writing the input of
    the next (the dependent launch must read x only after the previous kernel has written
    it)."""
    N = K = 1024
    c = workloads.q4_0_case(5, 1, N, K, bias=False)
    db = dev(c["blocks"])
    x0 = x_dev(c["x_bits"])
    wref = Q.dequantize(c["blocks"], K, "f32").astype(np.float64)
    for enable in (0, 1):
        old = w4.lib.w4_set_weight_prefetch(enable)
        try:
            ys = [x0]
            for _ in range(4):
                ys.append(w4.linear_q4_0(ys[-1], db))
            torch.cuda.synchronize()
            cur = c["x"].astype(np.float64)
            for i in range(1, 5):
                yr = cur @ wref.T
                bound = np.abs(cur) @ np.abs(wref).T
                got = ys[i].float().cpu().numpy().astype(np.float64)
                check(got, yr, bound, (enable, i))
                cur = got  # the next call's x is exactly this bf16 output
        finally:
            w4.lib.w4_set_weight_prefetch(old)


def test_q4_0_group32_reduction_on_device(w4):
    """Positive scales: the Q4_0 linear equals the group-32 linear on the same weight
    (scales d, signed codes c - 8), both within the tolerance of the one exact reference."""
    rng = np.random.default_rng(8)
    N, K = 96, 2048
    d = (np.abs(rng.standard_normal((N, K // 32))) * 0.01 + 1e-3).astype(np.float16).astype(np.float32)
    cq = rng.integers(0, 16, size=(N, K))
    blocks = Q.pack(d, cq)
    codes = O.pack_nibbles(cq - 8)
    xb, x = workloads.draw_x(rng, 1, K)
    yr, bound = Q.linear(x, blocks, K)
    y1 = w4.linear_q4_0(x_dev(xb), dev(blocks), out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    y2 = w4.linear(x_dev(xb), dev(codes), dev(d), K, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    check(y1, yr, bound, "q4_0")
    check(y2, yr, bound, "group-32")


@pytest.mark.parametrize("NK", [(1, 32), (3, 96), (17, 256), (64, 1056), (129, 4096)])
def test_q4_0_to_group32_bit_exact(w4, NK):
    # the re-laid-out codes and scales equal the oracle's, byte for byte (binary16 edge scales
    # included), with the codes written through the 16-byte path and through the byte path
    # (an output that starts one byte past a 16-byte boundary)
    N, K = NK
    blocks = special_blocks(N, K)
    codes_ref, scales_ref = Q.to_group32(blocks, K)
    db = dev(blocks)
    codes, scales = w4.q4_0_to_group32(db, K)
    assert np.array_equal(codes.cpu().numpy(), codes_ref), NK
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), scales_ref.view(np.uint32)), NK
    buf = torch.zeros(N * (K // 2) + 1, dtype=torch.uint8, device="cuda")
    c2 = buf[1:]
    s2 = torch.empty(N * (K // 32), dtype=torch.float32, device="cuda")
    w4.q4_0_to_group32(db, K, out=(c2, s2))
    assert np.array_equal(c2.cpu().numpy().reshape(N, K // 2), codes_ref), NK
    assert int(buf[0]) == 0


@pytest.mark.parametrize("case", [(1, 300, 4096), (1, 4096, 4096), (1, 17, 512), (16, 100, 1024), (33, 64, 2048)],
                         ids=lambda c: f"M{c[0]}_N{c[1]}_K{c[2]}")
def test_q4_0_group32_linear(w4, case):
    # the group-32 linear on the re-laid-out weight meets the Q4_0 oracle's tolerance
    M, N, K = case
    c = workloads.q4_0_case(M * 1000003 + N * 101 + K + 5, M, N, K)
    yr, bound = Q.linear(c["x"], c["blocks"], K, c["bias"])
    codes, scales = w4.q4_0_to_group32(dev(c["blocks"]), K)
    y = w4.linear(x_dev(c["x_bits"]), codes, scales, K, bias=dev(c["bias"]), out_dtype=torch.float32)
    check(y.cpu().numpy().astype(np.float64), yr, bound, (M, N, K, "group-32"))
    layer = w4.Linear(codes, scales, dev(c["bias"]), K) if M <= 16 else None
    if layer is not None:
        check(layer(x_dev(c["x_bits"]), out_dtype=torch.float32).cpu().numpy().astype(np.float64), yr, bound,
              (M, N, K, "Linear"))
