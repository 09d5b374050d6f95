"""GPU parity of w4_lora_merge (C ABI) against the LoRA-merge oracle: the re-quantized
codes and scales are bit-identical (the fp32 step order is part of the definition), in
place and out of place, for ranks 0 to 64, odd widths and partial groups; a non-finite merge
is reported."""

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


def lora_case(N, K, r, seed):
    c = workloads.linear_case(seed, 1, N, K, outliers=True, bias=False)
    q, s = O.quantize_rtn(c["W"])
    rng = np.random.default_rng([11, seed])
    b = (rng.standard_normal((N, r)) * 0.05).astype(np.float32)
    a = (rng.standard_normal((r, K)) * 0.05).astype(np.float32)
    return O.pack_nibbles(q), s, b, a


@pytest.mark.parametrize("NKr", [(1, 1, 1), (3, 7, 2), (37, 333, 3), (64, 4096, 16), (300, 1000, 8), (5, 96, 64),
                                 (9, 40, 0), (33, 129, 17), (70, 520, 40), (256, 1024, 16), (31, 127, 1)])
def test_lora_merge_bit_exact(w4, NKr):
    N, K, r = NKr
    codes, s, b, a = lora_case(N, K, r, N + K + r)
    c = 2.0 / max(r, 1)
    q2, s2 = O.lora_merge(codes, s, K, b, a, c)
    dc, ds = dev(codes), dev(s)
    co, so = w4.lora_merge(dc, ds, K, dev(b) if r else None, dev(a) if r else None, c)
    assert np.array_equal(co.cpu().numpy(), O.pack_nibbles(q2)), NKr
    assert np.array_equal(so.cpu().numpy().view(np.uint32), s2.view(np.uint32)), NKr
    # in place
    w4.lora_merge(dc, ds, K, dev(b) if r else None, dev(a) if r else None, c, out=(dc, ds))
    assert torch.equal(dc, co) and torch.equal(ds, so)


@pytest.mark.parametrize("NKr", [(2050, 4100, 16), (1024, 2048, 40), (4096, 4096, 0)])
def test_lora_merge_row_tile_walk(w4, NKr):
    # more 32-row tiles than a column tile's walkers: each CTA merges several row tiles in
    # turn (next tile's codes fetched ahead, the rank slices re-staged per chunk when r > 32)
    N, K, r = NKr
    codes, s, b, a = lora_case(N, K, r, 3 * N + K + r)
    c = 2.0 / max(r, 1)
    q2, s2 = O.lora_merge(codes, s, K, b, a, c)
    co, so = w4.lora_merge(dev(codes), dev(s), K, dev(b) if r else None, dev(a) if r else None, c)
    assert np.array_equal(co.cpu().numpy(), O.pack_nibbles(q2)), NKr
    assert np.array_equal(so.cpu().numpy().view(np.uint32), s2.view(np.uint32)), NKr


def test_lora_merge_full_size_in_place(w4):
    # the merge the bench times: rank 16 into (14336, 4096), in place, every code and scale
    N, K, r = 14336, 4096, 16
    codes, s, b, a = lora_case(N, K, r, 99)
    q2, s2 = O.lora_merge(codes, s, K, b, a, 2.0 / r)
    dc, ds = dev(codes), dev(s)
    w4.lora_merge(dc, ds, K, dev(b), dev(a), 2.0 / r, out=(dc, ds))
    assert np.array_equal(dc.cpu().numpy(), O.pack_nibbles(q2))
    assert np.array_equal(ds.cpu().numpy().view(np.uint32), s2.view(np.uint32))


def test_lora_merge_ties_and_near_ties(w4):
    # merged values on and 2^-22 beside half-integers of the new scale, with scales whose
    # reciprocal is exact in fp32 (1, 2^-20) and inexact (3, 3/8, 1/3, 5, 7): the codes round
    # half to even exactly as the oracle's division does
    from test_lora_oracle import lora_tie_case
    scales = [1.0, 3.0, 0.375, float(np.float32(1 / 3)), 5.0, 1.0, 2.0**-20, 7.0]
    codes, s, b, a, q, d = lora_tie_case(scales)
    q2, s2 = O.lora_merge(codes, s, 64, b, a, 1.0)
    co, so = w4.lora_merge(dev(codes), dev(s), 64, dev(b), dev(a), 1.0)
    assert np.array_equal(co.cpu().numpy(), O.pack_nibbles(q2))
    assert np.array_equal(so.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    unit = [i for i, v in enumerate(scales) if v == 1.0]
    expect = np.vectorize(lambda v: round(v))(q + d)[unit]
    assert np.array_equal(q2[unit].astype(np.int64), expect)


def test_lora_merge_worked_example_on_device(w4):
    g = read_golden("lora_merge_worked_example.txt")
    codes = np.array([int(t, 16) for t in g["codes_hex"]], np.uint8).reshape(1, 2)
    s = np.array([[float(g["scales"][0])]], np.float32)
    b = np.array([[float(v) for v in g["c2.b"]]], np.float32)
    a = np.array([[float(v) for v in g["c2.a0"]], [float(v) for v in g["c2.a1"]]], np.float32)
    co, so = w4.lora_merge(dev(codes), dev(s), 4, dev(b), dev(a), float(g["c2.c"][0]))
    q = np.array([[int(float(v)) for v in g["c2.q"]]], np.int8)
    assert np.array_equal(co.cpu().numpy(), O.pack_nibbles(q))
    assert so.cpu().numpy()[0, 0] == float(g["c2.s"][0])


def test_lora_merge_nonfinite_reported(w4):
    codes, s, b, a = lora_case(4, 64, 2, 1)
    b[2, 1] = np.inf
    with pytest.raises(Exception):
        w4.lora_merge(dev(codes), dev(s), 64, dev(b), dev(a), 1.0)
