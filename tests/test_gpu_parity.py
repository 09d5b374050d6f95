"""GPU parity: the CUDA library (called through its C ABI) against the CPU oracle on the
same seeded inputs. Codes, scales and dequantized weights must be bit-identical; linear
outputs must satisfy |y - y_ref| <= 4e-3 * sum_k |x w| + 1e-6 per element.

Small sizes span several tiles and ragged tails; the full sizes of the five workloads are
checked too (all outputs where the fp64 oracle is cheap, sampled activation rows for the
prefill GEMMs)."""

import math

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


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def x_dev(x_bits):
    return dev(x_bits.view(np.int16)).view(torch.bfloat16)


def y_host(y):
    return y.float().cpu().numpy().astype(np.float64)


def oracle_pack(W):
    q, s = O.quantize_rtn(W)
    return O.pack_nibbles(q), s


# ---------------------------------------------------------------------------
# quantize (a1 + a2)
# ---------------------------------------------------------------------------

QUANT_SHAPES = [(1, 1), (3, 5), (64, 33), (7, 4095), (33, 4096), (17, 1001), (256, 1000)]


@pytest.mark.parametrize("shape", QUANT_SHAPES)
def test_quantize_bit_exact(w4, shape):
    c = workloads.linear_case(100 + shape[1], 1, shape[0], shape[1], outliers=True)
    codes, scales = w4.quantize_rtn(dev(c["W"]))
    rc, rs = oracle_pack(c["W"])
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_quantize_config1_bit_exact(w4):
    c = workloads.config1()
    codes, scales = w4.quantize_rtn(dev(c["W"]))
    rc, rs = oracle_pack(c["W"])
    assert codes.shape == (256, 500) and scales.shape == (256, 32)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("NK", [(4096, 4095), (14336, 4096)])
def test_quantize_full_size_bit_exact(w4, NK):
    c = workloads.decode_case(*NK)
    codes, scales = w4.quantize_rtn(dev(c["W"]))
    rc, rs = oracle_pack(c["W"])
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_quantize_extremes_bit_exact(w4):
    """Huge, tiny, subnormal, zero groups and exact ties."""
    W = np.zeros((4, 70), np.float32)
    W[0, :8] = [7, 2.5, 3.5, -2.5, -0.5, 0.5, 1.5, -7]
    W[1, :5] = [3.4e38, -3.4e38, 1.0, 1e-30, -2e38]
    W[2, 32:37] = [1e-45, -1e-45, 7e-45, 3e-40, -1e-39]
    W[3, :] = np.float32(1e-3) * np.arange(70, dtype=np.float32)
    codes, scales = w4.quantize_rtn(dev(W))
    rc, rs = oracle_pack(W)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_quantize_rejects_nonfinite(w4):
    W = np.ones((5, 40), np.float32)
    W[3, 17] = np.nan
    with pytest.raises(w4.W4Error) as e:
        w4.quantize_rtn(dev(W))
    assert e.value.name == "NONFINITE"
    W[3, 17] = -np.inf
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    w4.quantize_rtn(dev(W), status=status)
    assert int(status.item()) == 4
    status.zero_()
    w4.quantize_rtn(dev(np.ones((5, 40), np.float32)), status=status)
    assert int(status.item()) == 0


# ---------------------------------------------------------------------------
# dequantize (a3 + a4)
# ---------------------------------------------------------------------------

DTYPES = [("bf16", torch.bfloat16), ("f16", torch.float16), ("f32", torch.float32), ("f64", torch.float64)]


def _compare_dequant(w4, codes, scales, K):
    for name, tdt in DTYPES:
        got = w4.dequantize(dev(codes), dev(scales), K, tdt).cpu()
        ref = O.dequantize(codes, scales, K, name)
        if name == "bf16":
            assert np.array_equal(got.view(torch.int16).numpy().view(np.uint16), ref), name
        else:
            a = got.numpy()
            assert a.dtype == ref.dtype
            assert np.array_equal(a.view(np.uint8), np.ascontiguousarray(ref).view(np.uint8)), name


@pytest.mark.parametrize("NK", [(1, 1), (3, 5), (64, 33), (9, 64), (5, 1000), (40, 4095), (8, 4096), (3, 100),
                                (129, 4095), (3, 20001)])
def test_dequant_bit_exact_all_dtypes(w4, NK):
    N, K = NK
    rng = np.random.default_rng(N * 1000 + K)
    # every byte value (v2 allows nibble 8), scales spanning normal and tiny magnitudes
    codes = rng.integers(0, 256, size=(N, (K + 1) // 2), dtype=np.uint8)
    if K % 2:
        codes[:, -1] &= 0x0F
    scales = (rng.uniform(0.5, 2.0, size=(N, (K + 31) // 32)) *
              10.0 ** rng.integers(-40, 30, size=(N, (K + 31) // 32))).astype(np.float32)
    scales = np.maximum(scales, np.float32(1e-45))
    _compare_dequant(w4, codes, scales, K)


def test_dequant_config2_odd_width_full_size(w4):
    """The odd-width dequant check of the decode workload: (4096, 4095)."""
    c = workloads.decode_case(4096, 4095)
    codes, scales = oracle_pack(c["W"])
    assert codes.shape == (4096, 2048) and scales.shape == (4096, 128)
    _compare_dequant(w4, codes, scales, 4095)


def test_dequant_unaligned_output(w4):
    """An output view starting at an odd element offset takes the generic path."""
    rng = np.random.default_rng(1)
    codes = rng.integers(0, 256, size=(6, 32), dtype=np.uint8)
    scales = rng.uniform(0.1, 1, size=(6, 2)).astype(np.float32)
    buf = torch.empty(6 * 64 + 1, dtype=torch.bfloat16, device="cuda")
    out = buf[1:].view(6, 64)
    dc, ds = dev(codes), dev(scales)  # keep the tensors alive across the call
    w4.dequantize(dc, ds, 64, torch.bfloat16, out=out)
    ref = O.dequantize(codes, scales, 64, "bf16")
    assert np.array_equal(out.cpu().view(torch.int16).numpy().view(np.uint16), ref)


def test_dequant_unaligned_codes(w4):
    """Codes starting one byte past a 16-byte boundary (odd width) take the generic path."""
    rng = np.random.default_rng(2)
    N, K = 7, 99
    P = (K + 1) // 2
    codes = rng.integers(0, 256, size=(N, P), dtype=np.uint8)
    codes[:, -1] &= 0x0F
    scales = rng.uniform(0.1, 1, size=(N, (K + 31) // 32)).astype(np.float32)
    buf = torch.zeros(N * P + 1, dtype=torch.uint8, device="cuda")
    buf[1:] = dev(codes.reshape(-1))
    dc = buf[1:].view(N, P)
    assert dc.data_ptr() % 16 == 1
    ds = dev(scales)
    for dt, name in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
        out = w4.dequantize(dc, ds, K, dt)
        ref = O.dequantize(codes, scales, K, name)
        got = out.cpu()
        if name == "bf16":
            assert np.array_equal(got.view(torch.int16).numpy().view(np.uint16), ref)
        else:
            assert np.array_equal(got.numpy().view(np.uint8), np.ascontiguousarray(ref).view(np.uint8))


# ---------------------------------------------------------------------------
# linear (a5), all M-dispatch paths
# ---------------------------------------------------------------------------

def _linear_check(w4, c, out_dtype=torch.bfloat16, rows=None):
    codes, scales = oracle_pack(c["W"])
    x = x_dev(c["x_bits"])
    bias = dev(c["bias"]) if c["bias"] is not None else None
    y = w4.linear(x, dev(codes), dev(scales), c["K"], bias=bias, out_dtype=out_dtype)
    torch.cuda.synchronize()
    yg = y_host(y)
    xs = c["x"] if rows is None else c["x"][rows]
    if rows is not None:
        yg = yg[rows]
    yr, bound = O.linear(xs, codes, scales, c["K"], c["bias"])
    ok, worst = O.check_linear(yg, yr, bound)
    assert ok, f"worst error/allowance = {worst}"
    return worst


@pytest.mark.parametrize("MNK", [(1, 300, 4096), (4, 256, 1000), (8, 2400, 2432), (33, 96, 4096)])
def test_prepared_linear_matches_linear(w4, MNK):
    """w4.Linear (weights checked once) computes the same y as w4.linear, bitwise."""
    M, N, K = MNK
    c = workloads.linear_case(M * 7 + N + K, M, N, K)
    codes, scales = oracle_pack(c["W"])
    dc, ds, db = dev(codes), dev(scales), dev(c["bias"])
    x = x_dev(c["x_bits"])
    layer = w4.Linear(dc, ds, db, K=K)
    for dt in (torch.bfloat16, torch.float32):
        y1 = w4.linear(x, dc, ds, K, bias=db, out_dtype=dt)
        y2 = layer(x, out_dtype=dt)
        out = torch.empty_like(y1)
        y3 = layer(x, out=out)
        assert y3.data_ptr() == out.data_ptr()
        assert torch.equal(y1, y2) and torch.equal(y1, y3)
    yr, bound = O.linear(c["x"], codes, scales, K, c["bias"])
    ok, worst = O.check_linear(y_host(layer(x)), yr, bound)
    assert ok, worst
    with pytest.raises(ValueError):
        layer(x.float())
    with pytest.raises(ValueError):
        layer(x[:, : K - 1].contiguous())


def test_linear_config1(w4):
    _linear_check(w4, workloads.config1())
    _linear_check(w4, workloads.config1(), out_dtype=torch.float32)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 16, 17, 31, 32, 64, 65, 128, 129])
@pytest.mark.parametrize("NK", [(200, 4096), (96, 4095), (24, 1024), (40, 33)])
def test_linear_small(w4, M, NK):
    c = workloads.linear_case(M * 7 + NK[1], M, NK[0], NK[1], outliers=True)
    _linear_check(w4, c)


@pytest.mark.parametrize("NK", workloads.DECODE_SHAPES)
def test_linear_decode_full_size(w4, NK):
    _linear_check(w4, workloads.decode_case(*NK))


@pytest.mark.parametrize("M", workloads.BATCHED_M)
def test_linear_batched_full_size(w4, M):
    N, K = workloads.BATCHED_SHAPE
    _linear_check(w4, workloads.decode_case(N, K, M=M, config=3, bias=True))


@pytest.mark.parametrize("MNK", workloads.PREFILL_SHAPES)
def test_linear_prefill_full_size_sampled(w4, MNK):
    M, N, K = MNK
    c = workloads.decode_case(N, K, M=M, config=4)
    rows = np.sort(np.random.default_rng(0).choice(M, 48, replace=False))
    _linear_check(w4, c, rows=rows)


def test_linear_exact_closed_form(w4):
    """Power-of-two scales and small-integer activations: every product and partial sum
    is exact in fp32, so an fp32 y must equal the oracle exactly and a bf16 y must be
    that exact value rounded once (RNE)."""
    rng = np.random.default_rng(12)
    for M, N, K in [(1, 64, 4096), (3, 40, 1000), (16, 128, 256), (200, 256, 512)]:
        vals = rng.integers(-8, 8, size=(N, K))
        codes = O.pack_nibbles(vals)
        scales = (2.0 ** rng.integers(-6, -3, size=(N, (K + 31) // 32))).astype(np.float32)
        xv = rng.integers(-2, 3, size=(M, K)).astype(np.float32)
        x_bits = O.f32_to_bf16_bits(xv)
        yr, _ = O.linear(xv, codes, scales, K)
        assert np.abs(yr).max() <= 256
        y = w4.linear(x_dev(x_bits), dev(codes), dev(scales), K, out_dtype=torch.float32)
        assert np.array_equal(y_host(y), yr), (M, N, K, "f32")
        y = w4.linear(x_dev(x_bits), dev(codes), dev(scales), K, out_dtype=torch.bfloat16)
        exp = O.f32_to_bf16_bits(yr.astype(np.float32))  # yr is exact in fp32 here
        assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), exp), (M, N, K, "bf16")


def test_linear_one_hot(w4):
    c = workloads.linear_case(3, 1, 64, 4096)
    codes, scales = oracle_pack(c["W"])
    wref = O.dequantize(codes, scales, 4096, "f32").astype(np.float64)
    for k in (0, 31, 32, 4095):
        x = np.zeros((1, 4096), np.float32)
        x[0, k] = 1.0
        y = w4.linear(x_dev(O.f32_to_bf16_bits(x)), dev(codes), dev(scales), 4096, out_dtype=torch.float32)
        assert np.array_equal(y_host(y)[0], wref[:, k])


def test_linear_zero_rows(w4):
    """All-zero weight rows (floor scales, codes 0) give y = bias exactly."""
    c = workloads.linear_case(4, 3, 48, 512)
    c["W"][5] = 0
    c["W"][17] = 0
    codes, scales = oracle_pack(c["W"])
    y = w4.linear(x_dev(c["x_bits"]), dev(codes), dev(scales), 512, bias=dev(c["bias"]), out_dtype=torch.float32)
    yh = y_host(y)
    assert np.array_equal(yh[:, 5], np.full(3, np.float64(c["bias"][5])))
    assert np.array_equal(yh[:, 17], np.full(3, np.float64(c["bias"][17])))


# ---------------------------------------------------------------------------
# decode GEMV (M = 1): TMA stage ring, ragged row blocks and k-tiles, deep rows, launch
# overlap (programmatic dependent launch with weight prefetch)
# ---------------------------------------------------------------------------

DECODE_EDGE_NK = [(1, 128), (16, 256), (17, 384), (33, 640), (2368, 2048), (2400, 2432), (4100, 4096),
                  (5000, 1152), (300, 14336), (64, 28672),
                  # K a multiple of 1024 (whole-stage boxes): one row, odd row counts, a row
                  # count just above two per CTA slot, rows of 4, 12 and 36 k-tiles
                  (1, 1024), (3, 3072), (593, 1024), (2049, 3072), (7, 9216)]


@pytest.mark.parametrize("NK", DECODE_EDGE_NK)
def test_linear_decode_edges(w4, NK):
    N, K = NK
    c = workloads.linear_case(N + 3 * K, 1, N, K, outliers=True)
    _linear_check(w4, c)
    _linear_check(w4, c, out_dtype=torch.float32)


@pytest.mark.parametrize("M", [2, 3, 7, 8, 9, 13, 16])
@pytest.mark.parametrize("NK", [(2400, 2432), (300, 14336), (33, 1152)])
def test_linear_small_m_tensor_core_path(w4, M, NK):
    """Small M on the TMA-fed tensor-core kernel (activation rows as MMA columns): ragged
    row blocks and k-tiles, one and two n-tiles, activations up to shared-memory size."""
    N, K = NK
    c = workloads.linear_case(M * 31 + N + K, M, N, K, outliers=True)
    _linear_check(w4, c)
    _linear_check(w4, c, out_dtype=torch.float32)


@pytest.mark.parametrize("special", ["tiny", "huge", "subnormal", "none"])
def test_linear_decode_activation_range(w4, special):
    """Activations at the edges of the bf16 range on the M = 1 decode path: finer than
    fp16's subnormal spacing, beyond fp16's range, bf16 subnormals, or none of those."""
    N, K = 600, 4096
    c = workloads.linear_case(4242, 1, N, K)
    codes, scales = oracle_pack(c["W"])
    xb = c["x_bits"].copy()
    if special == "tiny":      # 2^-20 * 1.5: exact in bf16, not in fp16
        xb[0, 17] = np.float32(1.5 * 2.0 ** -20).view(np.uint32) >> 16
    elif special == "huge":    # 2^17: beyond fp16's largest finite value
        xb[0, 4000] = np.float32(2.0 ** 17).view(np.uint32) >> 16
    elif special == "subnormal":
        xb[0, 100] = 0x0003
    x = O.bf16_bits_to_f32(xb).astype(np.float64)
    y = w4.linear(x_dev(xb), dev(codes), dev(scales), K, bias=dev(c["bias"]), out_dtype=torch.float32)
    yr, bound = O.linear(x, codes, scales, K, c["bias"])
    ok, worst = O.check_linear(y_host(y), yr, bound)
    assert ok, worst


def test_linear_decode_unaligned_x(w4):
    """x starting 8 bytes past a 16-byte boundary takes another kernel; same result."""
    c = workloads.linear_case(77, 1, 300, 2048)
    codes, scales = oracle_pack(c["W"])
    buf = torch.zeros(2048 + 8, dtype=torch.bfloat16, device="cuda")
    buf[4:4 + 2048] = x_dev(c["x_bits"])[0]
    x = buf[4:4 + 2048].view(1, 2048)
    assert x.data_ptr() % 16 == 8
    y = w4.linear(x, dev(codes), dev(scales), 2048, bias=dev(c["bias"]))
    yr, bound = O.linear(c["x"], codes, scales, 2048, c["bias"])
    ok, worst = O.check_linear(y_host(y), yr, bound)
    assert ok, worst


def _chain(w4, layers, x0, graph):
    """y_i = linear(y_{i-1}) for alternating weights on one stream, no host sync between
    layers; optionally captured once into a CUDA graph and replayed."""
    outs = [torch.empty((1, layers[i % 2][2].shape[0]), dtype=torch.bfloat16, device="cuda") for i in range(6)]

    def run():
        x = x0
        for i in range(6):
            codes, scales, bias = layers[i % 2][1:]
            w4.linear(x, codes, scales, x.shape[1], bias=bias, out=outs[i])
            x = outs[i]

    if graph:
        run()  # warm-up outside capture (tensor maps, attributes)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        for o in outs:
            o.zero_()
        g.replay()
        g.replay()
    else:
        run()
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("prefetch", [False, True])
@pytest.mark.parametrize("graph", [False, True])
def test_linear_decode_chain_launch_overlap(w4, prefetch, graph):
    """Each layer reads the previous layer's output: the kernel must not read x (nor write
    y) before the previous kernel has finished, with and without weight prefetch."""
    K = 2048
    layers = []
    for i in range(2):
        c = workloads.linear_case(500 + i, 1, K, K)
        codes, scales = oracle_pack(c["W"])
        layers.append((c, dev(codes), dev(scales), dev(c["bias"])))
    torch.cuda.synchronize()
    prev = w4.set_weight_prefetch(prefetch)
    try:
        x0 = x_dev(workloads.linear_case(600, 1, 8, K)["x_bits"])
        outs = _chain(w4, layers, x0, graph)
    finally:
        w4.set_weight_prefetch(prev)
    x = x0
    for i, y in enumerate(outs):
        c = layers[i % 2][0]
        xb = x.cpu().view(torch.int16).numpy().view(np.uint16)
        yr, bound = O.linear(O.bf16_bits_to_f32(xb).astype(np.float64), layers[i % 2][1].cpu().numpy(),
                             layers[i % 2][2].cpu().numpy(), K, c["bias"])
        ok, worst = O.check_linear(y_host(y), yr, bound)
        assert ok, (i, worst)
        x = y
    assert w4.device_error() == "OK"


# ---------------------------------------------------------------------------
# asymmetric act-order (a6)
# ---------------------------------------------------------------------------

def _asym_data(c):
    u, s, z = O.quantize_asym_minmax(c["W"], c["g_idx"], c["n_groups"])
    return O.pack_nibbles(u), s, z


def _asym_check(w4, c, prepared, rows=None):
    codes, s, z = _asym_data(c)
    gi = dev(c["g_idx"])
    dcodes = dev(codes)
    perm = None
    if prepared:
        dcodes, perm = w4.asym_prepare(dcodes, gi, c["K"], c["n_groups"])
        assert np.array_equal(perm.cpu().numpy(), np.argsort(c["g_idx"], kind="stable"))
    y = w4.linear_asym_gidx(x_dev(c["x_bits"]), dcodes, dev(s), dev(z), gi, perm=perm, bias=dev(c["bias"]))
    yg = y_host(y)
    xs = c["x"]
    if rows is not None:
        yg, xs = yg[rows], xs[rows]
    yr, bound = O.linear_asym_gidx(xs, codes, s, z, c["g_idx"], c["K"], c["bias"])
    ok, worst = O.check_linear(yg, yr, bound)
    assert ok, f"worst error/allowance = {worst}"


@pytest.mark.parametrize("prepared", [False, True])
@pytest.mark.parametrize("M", [1, 2, 4, 5, 16, 33])
@pytest.mark.parametrize("NKG", [(72, 512, 128), (40, 1024, 64), (24, 4095, 128), (16, 96, 32)])
def test_asym_small(w4, prepared, M, NKG):
    N, K, group = NKG
    c = workloads.asym_case(M=M, N=N, K=K, group=group, seed=M * 31 + K)
    _asym_check(w4, c, prepared)


@pytest.mark.parametrize("M", [1, 3, 9, 16, 33])
@pytest.mark.parametrize("NK", [(48, 512), (40, 1280)])
def test_asym_ragged_groups(w4, M, NK):
    """Act-order groups of uneven sizes (g_idx drawn at random, not a permutation of equal
    groups): after sorting, group boundaries fall inside 32-column chunks, which the
    tensor-core path handles column by column."""
    N, K = NK
    c = workloads.asym_case(M=M, N=N, K=K, group=128, seed=900 + M + K)
    n_groups = 7
    c["g_idx"] = np.random.default_rng(M + K).integers(0, n_groups, size=K).astype(np.int32)
    c["n_groups"] = n_groups
    _asym_check(w4, c, prepared=True)
    _asym_check(w4, c, prepared=False)


@pytest.mark.parametrize("K", [16384, 16512])
def test_asym_one_row_long(w4, K):
    """One activation row at the longest width the decode kernel gathers itself (16384)
    and just past it (gathered once into the workspace instead)."""
    c = workloads.asym_case(M=1, N=40, K=K, group=128, seed=K)
    _asym_check(w4, c, prepared=True)


@pytest.mark.parametrize("M", workloads.ASYM_M)
def test_asym_full_size(w4, M):
    c = workloads.asym_case(M=M)
    rows = None if M <= 16 else np.sort(np.random.default_rng(1).choice(M, 48, replace=False))
    _asym_check(w4, c, prepared=True, rows=rows)


def test_asym_prepare_reorders_codes(w4):
    c = workloads.asym_case(M=1, N=10, K=77, group=16, seed=3)
    codes, s, z = _asym_data(c)
    out, perm = w4.asym_prepare(dev(codes), dev(c["g_idx"]), 77, c["n_groups"])
    p = np.argsort(c["g_idx"], kind="stable")
    u = O.unpack_unsigned(codes, 77)
    assert np.array_equal(out.cpu().numpy(), O.pack_nibbles(u[:, p]))
    assert np.array_equal(perm.cpu().numpy(), p)


def test_asym_prepare_rejects_bad_gidx(w4):
    gi = np.zeros(64, np.int32)
    gi[5] = 4
    with pytest.raises(w4.W4Error) as e:
        w4.asym_prepare(dev(np.zeros((2, 32), np.uint8)), dev(gi), 64, 4)
    assert e.value.name == "GIDX"


def test_asym_float_gidx_accepted(w4):
    """Keras stores g_idx as float32; the binding casts it (exact below 2**24)."""
    c = workloads.asym_case(M=2, N=16, K=256, group=64, seed=8)
    codes, s, z = _asym_data(c)
    y1 = w4.linear_asym_gidx(x_dev(c["x_bits"]), dev(codes), dev(s), dev(z), dev(c["g_idx"]))
    y2 = w4.linear_asym_gidx(x_dev(c["x_bits"]), dev(codes), dev(s), dev(z),
                             dev(c["g_idx"].astype(np.float32)))
    assert torch.equal(y1, y2)


# ---------------------------------------------------------------------------
# validation (LoopQ validate rules) on the device
# ---------------------------------------------------------------------------

def test_validate_rules_gpu(w4):
    K, N = 5, 2
    codes = O.pack_nibbles(np.array([[1, -1, 7, -7, 0], [0, 1, 2, 3, 4]]))
    s = np.ones((N, 1), np.float32)
    assert w4.validate(dev(codes), dev(s), K, 2) == "OK"
    assert w4.validate(dev(codes), dev(s), K, 1) == "OK"
    assert w4.validate(dev(codes), dev(s), K, 3) == "VERSION"
    for bad in (0.0, -1.0, np.nan, np.inf):
        s2 = s.copy()
        s2[1, 0] = bad
        assert w4.validate(dev(codes), dev(s2), K, 2) == O.validate(codes, s2, K, 2) == "SCALE"
    c2 = codes.copy()
    c2[0, -1] |= 0x10
    assert w4.validate(dev(c2), dev(s), K, 2) == "HIGH_NIBBLE"
    c3 = codes.copy()
    c3[1, 0] = 0x80
    assert w4.validate(dev(c3), dev(s), K, 2) == "OK"
    assert w4.validate(dev(c3), dev(s), K, 1) == "RESERVED_CODE"


def test_validate_brute_force_256(w4):
    allb = np.arange(256, dtype=np.uint8).reshape(256, 1)
    one = np.ones((1, 1), np.float32)
    v1 = [b for b in range(256) if w4.validate(dev(allb[b:b + 1]), dev(one), 2, 1) == "RESERVED_CODE"]
    odd = [b for b in range(256) if w4.validate(dev(allb[b:b + 1]), dev(one), 1, 2) == "HIGH_NIBBLE"]
    assert len(v1) == 31 and len(odd) == 240


def test_validate_asym_rules_gpu(w4):
    K, N, G = 6, 2, 2
    codes = O.pack_nibbles(np.arange(12).reshape(N, K))
    s = np.ones((N, G), np.float32)
    z = np.full((N, G), 8, np.int8)
    gi = np.array([0, 1, 0, 1, 1, 0], np.int32)
    assert w4.validate_asym(dev(codes), dev(s), dev(z), dev(gi), K) == "OK"
    z2 = z.copy()
    z2[1, 1] = 16
    assert w4.validate_asym(dev(codes), dev(s), dev(z2), dev(gi), K) == "ZERO"
    gi2 = gi.copy()
    gi2[3] = 2
    assert w4.validate_asym(dev(codes), dev(s), dev(z), dev(gi2), K) == "GIDX"
    s2 = s.copy()
    s2[0, 1] = -2
    assert w4.validate_asym(dev(codes), dev(s2), dev(z), dev(gi), K) == "SCALE"


def test_device_error_clear(w4):
    assert w4.device_error() == "OK"
