"""The bias gradient without a caller workspace (fp8_dbias_noalloc).

Some callers cannot allocate device memory -- code running under a memory
manager it does not control, such as a plugin in a serving runtime with a fixed
device-memory budget -- so they have no workspace to hand to fp8_dbias.  This
entry point runs the same kernel with its scratch in a fixed 1 MiB array inside
the library.  The test calls it through the C ABI twice in a row and checks each
result against fp8_dbias (with a workspace) on the same input, and against the
CPU oracle's column sums, within the bias gradient tolerance the other tests
use: max(1 bf16 ulp, 2e-6 sum|g|).  It also checks that a request beyond the
fixed scratch is refused.  This file is collected last so a stopped run has
already run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def bf16_ulp(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, np.ldexp(1.0, (e - 7).astype(np.int64)), np.ldexp(1.0, -133))


def check_close(got, want, g):
    got = got.float().cpu().double().numpy()
    want = want.float().cpu().double().numpy()
    sa = g.double().abs().sum(0).cpu().numpy()
    tol = np.maximum(bf16_ulp(want), 2e-6 * sa)
    assert np.all(np.abs(got - want) <= tol), np.max(np.abs(got - want) / tol)


def check_oracle(got, g_np, dtype, M, N, sg=1.0):
    """got (bf16 device tensor) vs the oracle's fixed-order fp32 column sums."""
    want, _, sa = oracle.dbias(g_np, dtype, M, N, sg)
    gv = oracle.bf16_to_f32(got.cpu().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    ov = oracle.bf16_to_f32(want).astype(np.float64)
    tol = np.maximum(oracle.bf16_ulp(ov), 2e-6 * sa)
    assert np.all(np.abs(gv - ov) <= tol), np.max(np.abs(gv - ov) / tol)


def test_dbias_noalloc_matches_workspace_entry_point():
    import fp8_delayed_scaling_03_b200 as F
    lib = F._lib
    stream = torch.cuda.current_stream().cuda_stream
    for i, (M, N) in enumerate([(2048, 1024), (4096, 11008)]):
        g = wl.normal((M, N), 1e-3 * (1 + i), 5151 + i).cuda()
        ref = torch.empty(N, dtype=torch.bfloat16, device="cuda")
        out = torch.full((N,), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(F.fp8_dbias_workspace_bytes(M, N), dtype=torch.uint8, device="cuda")
        assert lib.fp8_dbias(g.data_ptr(), F.FP8_DT_BF16, M, N, N, None, ref.data_ptr(), ws.data_ptr(),
                             ws.numel(), stream) == 0
        assert lib.fp8_dbias_noalloc(g.data_ptr(), F.FP8_DT_BF16, M, N, N, None, out.data_ptr(), stream) == 0
        torch.cuda.synchronize()
        check_close(out, ref, g)
        if i == 0:
            check_oracle(out, g.cpu().view(torch.int16).numpy().view(np.uint16), oracle.DT_BF16, M, N)
    # fp8 g with its scale (dequantized before the sum), two calls in a row
    M, N = 3000, 700
    codes = torch.randint(0, 0x5C, (M, 704), dtype=torch.int32).to(torch.uint8)
    codes[:, N:] = 0
    g8 = codes.cuda()[:, :N]
    sg = torch.tensor([37.5], device="cuda")
    ws = torch.zeros(F.fp8_dbias_workspace_bytes(M, N), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        ref = torch.empty(N, dtype=torch.bfloat16, device="cuda")
        out = torch.empty(N, dtype=torch.bfloat16, device="cuda")
        assert lib.fp8_dbias(g8.data_ptr(), F.FP8_DT_E5M2, M, N, 704, sg.data_ptr(), ref.data_ptr(), ws.data_ptr(),
                             ws.numel(), stream) == 0
        assert lib.fp8_dbias_noalloc(g8.data_ptr(), F.FP8_DT_E5M2, M, N, 704, sg.data_ptr(), out.data_ptr(),
                                     stream) == 0
        torch.cuda.synchronize()
        deq = g8.cpu().view(torch.float8_e5m2).double() / 37.5
        check_close(out, ref, deq)
        check_oracle(out, np.ascontiguousarray(codes.numpy()), oracle.DT_E5M2, M, N, 37.5)
    # beyond the fixed scratch: refused, nothing enqueued
    big_n = 1 << 20
    assert F.fp8_dbias_workspace_bytes(2048, big_n) > (1 << 20)
    assert lib.fp8_dbias_noalloc(ctypes.c_void_p(g.data_ptr()), F.FP8_DT_BF16, 2048, big_n, big_n, None,
                                 ctypes.c_void_p(out.data_ptr()), stream) == F.FP8_ERR_TOO_LARGE
    assert F.fp8_get_device_status() == 0
