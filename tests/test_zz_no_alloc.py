"""The act-order linear entry point that allocates nothing (w4_linear_asym_gidx_noalloc).

Its callers are host programs that may not allocate device memory at call time, so the
library keeps the scratch memory (activations gathered into sorted column order) in a fixed
16 MiB array of its own. This test calls that entry point through the C ABI twice in a row
on different activations -- the second call reuses the array the first one filled -- and
checks each result against the regular entry point (which takes a caller-provided workspace)
and the CPU oracle, with the linear tolerance of the other tests. It also checks the size
limit. The file sorts last so that a run stopping at the first failure has already run every
other test; it passes alone in a fresh process as well (the first call does the set-up)."""

import ctypes

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


def test_noalloc_matches_workspace_entry_point_twice(w4):
    M, N, K, group = 96, 320, 2048, 128  # M above the decode sizes: the scratch-using GEMM path
    case = workloads.asym_case(M=M, N=N, K=K, group=group, seed=77)
    u, s, z = O.quantize_asym_minmax(case["W"], case["g_idx"], case["n_groups"])
    codes = O.pack_nibbles(u)
    g_idx = _dev(case["g_idx"])
    sorted_codes, perm = w4.asym_prepare(_dev(codes), g_idx, K, case["n_groups"])
    ds, dz, db = _dev(s), _dev(z), _dev(case["bias"])
    assert w4.asym_workspace_bytes(M, N, K, case["n_groups"]) > 0
    rng = np.random.default_rng(5)
    for call in range(2):
        x_bits, x = workloads.bf16_round(rng.standard_normal((M, K), dtype=np.float32))
        xd = _dev(x_bits.view(np.int16)).view(torch.bfloat16)
        y_na = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        st = w4.lib.w4_linear_asym_gidx_noalloc(
            w4._ptr(xd), M, w4._ptr(sorted_codes), w4._ptr(ds), w4._ptr(dz), w4._ptr(g_idx), w4._ptr(perm),
            N, K, case["n_groups"], w4._ptr(db), w4._ptr(y_na), 0, w4._stream())
        assert st == 0, w4.STATUS[st]
        y_ws = w4.linear_asym_gidx(xd, sorted_codes, ds, dz, g_idx, perm=perm, bias=db)
        torch.cuda.synchronize()
        yr, bound = O.linear_asym_gidx(x, codes, s, z, case["g_idx"], K, case["bias"])
        a = y_na.float().cpu().numpy().astype(np.float64)
        b = y_ws.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(a - b) <= 4e-3 * bound + 1e-6), f"call {call}: differs from the workspace entry point"
        ok, worst = O.check_linear(a, yr, bound)
        assert ok, f"call {call}: worst error/allowance {worst}"
    assert w4.device_error() == "OK"


def test_noalloc_rejects_shapes_above_its_scratch(w4):
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: the size check fails first
    # 4096 x 4096 bf16 activations need 32 MiB of scratch, above the 16 MiB array; 2049 rows
    # are the first row count above it at K = 4096; the limit holds whichever kernel would
    # serve the shape (n_groups = 3 here keeps it off the tensor-core path)
    for M, n_groups in [(4096, 32), (2049, 32), (2049, 3), (1 << 40, 32)]:
        st = w4.lib.w4_linear_asym_gidx_noalloc(fake, M, fake, fake, fake, fake, fake, 256, 4096, n_groups, None,
                                                fake, 0, None)
        assert w4.STATUS[st] == "SHAPE", (M, n_groups)


def test_noalloc_at_its_limit(w4):
    """M = 2048 at K = 4096 (the act-order prefill shape, N = 11008, 32 groups of 128) needs
    exactly the 16 MiB of the array: accepted, equal to the workspace entry point on every
    output and to the oracle on sampled activation rows."""
    a = workloads.asym_random_codes(2048)
    M, N, K, G = a["M"], a["N"], a["K"], a["n_groups"]
    assert M * K * 2 == 16 << 20
    g_idx = _dev(a["g_idx"])
    sorted_codes, perm = w4.asym_prepare(_dev(a["codes"]), g_idx, K, G)
    ds, dz, db = _dev(a["scales"]), _dev(a["zeros"]), _dev(a["bias"])
    xd = _dev(a["x_bits"].view(np.int16)).view(torch.bfloat16)
    y_na = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = w4.lib.w4_linear_asym_gidx_noalloc(
        w4._ptr(xd), M, w4._ptr(sorted_codes), w4._ptr(ds), w4._ptr(dz), w4._ptr(g_idx), w4._ptr(perm),
        N, K, G, w4._ptr(db), w4._ptr(y_na), 0, w4._stream())
    assert st == 0, w4.STATUS[st]
    y_ws = w4.linear_asym_gidx(xd, sorted_codes, ds, dz, g_idx, perm=perm, bias=db)
    torch.cuda.synchronize()
    rows = np.random.default_rng(2048).choice(M, 24, replace=False)
    yr, bound = O.linear_asym_gidx(a["x"][rows], a["codes"], a["scales"], a["zeros"], a["g_idx"], K, a["bias"])
    na = y_na.float().cpu().numpy().astype(np.float64)
    ws = y_ws.float().cpu().numpy().astype(np.float64)
    assert np.array_equal(na, ws), "the two entry points run the same kernels on the same inputs"
    ok, worst = O.check_linear(na[rows], yr, bound)
    assert ok, worst
    assert w4.device_error() == "OK"
