"""Failure detection on the GPU without a fault: a bounded device wait is made to expire
(w4_selftest_wait_timeout: one CTA waits on a barrier that nothing arrives on, with a 2 ms
limit), the host reads W4_ERR_TIMEOUT through w4_device_error(), the read clears it, and the
context stays usable -- the next linear call runs and matches the oracle."""

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


def test_expired_wait_reports_timeout_and_clears(w4):
    assert w4.device_error() == "OK"
    w4.selftest_wait_timeout(2_000_000)
    assert w4.device_error() == "TIMEOUT"
    assert w4.device_error() == "OK"  # reading the word cleared it


def test_context_usable_after_timeout(w4):
    w4.selftest_wait_timeout(1_000_000)
    assert w4.device_error() == "TIMEOUT"
    c = workloads.linear_case(909, 1, 300, 2048)
    q, s = O.quantize_rtn(c["W"])
    codes = O.pack_nibbles(q)
    x = _dev(c["x_bits"].view(np.int16)).view(torch.bfloat16)
    y = w4.linear(x, _dev(codes), _dev(s), 2048, bias=_dev(c["bias"]), out_dtype=torch.float32)
    yr, bound = O.linear(c["x"], codes, s, 2048, c["bias"])
    ok, worst = O.check_linear(y.cpu().numpy().astype(np.float64), yr, bound)
    assert ok, worst
    assert w4.device_error() == "OK"


def test_timeout_on_a_stream_then_work_on_it(w4):
    """The expired wait on a side stream does not disturb later work queued on that stream."""
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        w4.selftest_wait_timeout(500_000)
        c = workloads.linear_case(910, 3, 256, 1024)
        q, s = O.quantize_rtn(c["W"])
        codes = O.pack_nibbles(q)
        x = _dev(c["x_bits"].view(np.int16)).view(torch.bfloat16)
        y = w4.linear(x, _dev(codes), _dev(s), 1024, out_dtype=torch.float32)
    side.synchronize()
    assert w4.device_error() == "TIMEOUT"
    yr, bound = O.linear(c["x"], codes, s, 1024)
    ok, worst = O.check_linear(y.cpu().numpy().astype(np.float64), yr, bound)
    assert ok, worst
