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
    # 4096 x 4096 bf16 activations need 32 MiB of scratch, above the 16 MiB array
    st = w4.lib.w4_linear_asym_gidx_noalloc(fake, 4096, fake, fake, fake, fake, fake, 256, 4096, 32, None, fake,
                                            0, None)
    assert w4.STATUS[st] == "SHAPE"
