"""The bounded waits on the GPU, made to run out on purpose: a flag that
nothing sets and an mbarrier that nothing arrives on, each with a 20 ms
limit (fp8_wait_selftest).  Each wait records FP8_ERR_DEVICE_TIMEOUT, the
kernel returns, the status read clears the word, and the context stays
usable: a quantize right afterwards matches the oracle bit for bit.  No GPU
fault, trap or hang is involved."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import assert_codes_equal, bits, fp8_buffer, host_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def test_waits_run_out_and_report(fp8):
    assert fp8.fp8_get_device_status() == 0
    flag = torch.zeros(4, dtype=torch.int32, device="cuda")
    res = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    fp8.fp8_wait_selftest(flag, 20_000_000, res)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert res.tolist() == [0, 0]
    assert elapsed >= 0.02 and elapsed < 10.0, elapsed
    assert fp8.fp8_get_device_status() == fp8.FP8_ERR_DEVICE_TIMEOUT
    assert fp8.fp8_get_device_status() == 0           # the read cleared it
    flag.fill_(1)                                     # a flag that is set: that wait succeeds at once
    fp8.fp8_wait_selftest(flag, 20_000_000, res)
    torch.cuda.synchronize()
    assert res.tolist() == [1, 0]
    assert fp8.fp8_get_device_status() == fp8.FP8_ERR_DEVICE_TIMEOUT
    # the context is still usable
    x = wl.normal((512, 384), 1.0, 5151)
    ring, oring = fp8.ScaleRing(16), oracle.Ring(16)
    out = fp8_buffer(512, 384)
    fp8.fp8_quantize(x.cuda(), fp8.FP8_E4M3, ring.buf, 16, out)
    torch.cuda.synchronize()
    q, _, _ = oracle.quantize(bits(x), oracle.DT_BF16, oracle.E4M3, oring)
    assert_codes_equal(host_rows(out), q, oracle.E4M3)
    assert fp8.fp8_get_device_status() == 0
