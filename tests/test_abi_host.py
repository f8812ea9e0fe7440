"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/fp8lin.h, and rejects bad arguments before enqueuing any
work (so no CUDA call is reached here).  Pointers passed are fake aligned
addresses; validation never dereferences them."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def header_functions():
    src = open(os.path.join(ROOT, "include", "fp8lin.h")).read()
    return re.findall(r"FP8LIN_API\s+[\w\s\*]+?\b(fp8_\w+)\s*\(", src)


def test_exports_every_header_symbol(fp8):
    names = header_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(fp8._lib, n), n
        assert n in fp8.EXPORTED, n
    assert set(fp8.EXPORTED) == set(names)


def test_version_and_status_strings(fp8):
    assert "sm_100a" in fp8.fp8_version()
    for s in (0, -1, -2, -3, -5, -6, -7):
        assert fp8.fp8_status_string(s)
    assert fp8.fp8_status_string(12345) == "unknown status"


def test_ring_bytes(fp8):
    assert fp8.fp8_ring_bytes(16) == 80
    assert fp8.fp8_ring_bytes(1) == 20
    assert fp8.fp8_ring_bytes(0) == 0
    assert fp8.fp8_ring_bytes(4097) == 0


A = 0x100000  # a fake 16-byte aligned device address


def q(fp8, **kw):
    a = dict(inp=A, dt=fp8.FP8_DT_BF16, rows=4, cols=32, ld_in=32, fmt=0, ring=A + 0x1000, H=16,
             out=A + 0x2000, ld_out=32)
    a.update(kw)
    return fp8._lib.fp8_quantize(a["inp"], a["dt"], a["rows"], a["cols"], a["ld_in"], a["fmt"], a["ring"], a["H"],
                                 a["out"], a["ld_out"], None, None, None)


def test_quantize_validation(fp8):
    E = fp8
    assert q(fp8, inp=None) == E.FP8_ERR_INVALID_ARG
    assert q(fp8, ring=None) == E.FP8_ERR_INVALID_ARG                # current scaling needs amax_out
    assert q(fp8, out=None) == E.FP8_ERR_INVALID_ARG
    assert q(fp8, dt=E.FP8_DT_E4M3) == E.FP8_ERR_INVALID_ARG       # fp8 input is not quantized again
    assert q(fp8, dt=9) == E.FP8_ERR_INVALID_ARG
    assert q(fp8, fmt=2) == E.FP8_ERR_INVALID_ARG
    assert q(fp8, H=0) == E.FP8_ERR_INVALID_ARG
    assert q(fp8, ld_in=31) == E.FP8_ERR_INVALID_ARG
    assert q(fp8, ld_out=40) == E.FP8_ERR_MISALIGNED
    assert q(fp8, out=A + 8) == E.FP8_ERR_MISALIGNED
    assert q(fp8, ring=A + 2) == E.FP8_ERR_INVALID_ARG
    assert q(fp8, inp=A + 1) == E.FP8_ERR_INVALID_ARG            # bf16 must be 2-byte aligned
    assert q(fp8, rows=-1) == E.FP8_ERR_INVALID_ARG
    # zero sizes: accepted, nothing enqueued
    assert q(fp8, rows=0) == E.FP8_OK
    assert q(fp8, cols=0, ld_in=0, ld_out=0) == E.FP8_OK


def mm(fp8, **kw):
    a = dict(m=128, n=128, k=128, a=A, fmt_a=0, a_major=0, lda=128, b=A + 0x10000, fmt_b=0, b_major=0, ldb=128,
             scale_a=A + 0x20000, scale_b=A + 0x20010, bias=None, bias_dtype=0, bias_scale=None, d=A + 0x30000,
             ldd=128)
    a.update(kw)
    args = fp8.MmArgs(**a)
    return fp8._lib.fp8_mm(ctypes.byref(args), None)


def mmb(fp8, batch, sa, sb, sd, **kw):
    a = dict(m=128, n=128, k=128, a=A, fmt_a=0, a_major=0, lda=128, b=A + 0x10000, fmt_b=0, b_major=0, ldb=128,
             scale_a=A + 0x20000, scale_b=A + 0x20010, bias=None, bias_dtype=0, bias_scale=None, d=A + 0x30000,
             ldd=128)
    a.update(kw)
    args = fp8.MmArgs(**a)
    return fp8._lib.fp8_mm_batched(ctypes.byref(args), batch, sa, sb, sd, None)


def test_mm_batched_validation(fp8):
    """Checked before anything is enqueued (no GPU needed)."""
    E = fp8
    big = 128 * 128
    assert mmb(fp8, -1, big, big, big) == E.FP8_ERR_INVALID_ARG
    assert mmb(fp8, 2, -16, big, big) == E.FP8_ERR_INVALID_ARG
    assert mmb(fp8, 2, big + 8, big, big) == E.FP8_ERR_MISALIGNED         # fp8 batch stride: 16-byte multiple
    assert mmb(fp8, 2, big, 24, big) == E.FP8_ERR_MISALIGNED
    assert mmb(fp8, 2, big, big, big - 1) == E.FP8_ERR_INVALID_ARG        # outputs of two batches overlap
    assert mmb(fp8, 2, big, big, 0) == E.FP8_ERR_INVALID_ARG
    assert mmb(fp8, 0, big, big, big) == E.FP8_OK                         # empty batch: nothing enqueued
    assert mmb(fp8, 3, 0, 0, big, m=0) == E.FP8_OK
    assert mmb(fp8, 2, big, big, big, scale_a=None) == E.FP8_ERR_INVALID_ARG


def test_quantize_ex_and_ring_finalize_validation(fp8):
    E = fp8
    f = fp8._lib
    qa = fp8.QuantizeArgs(A, 0, 4, 32, 32, 0, A + 0x1000, 16, A + 0x2000, 32, None, None)
    qn = fp8.QuantizeArgs(A, 0, 4, 32, 32, 0, None, 16, A + 0x2000, 32, A + 0x3000, None)
    assert f.fp8_quantize_ex(ctypes.byref(qa), 2, None) == E.FP8_ERR_INVALID_ARG          # unknown flag
    assert f.fp8_quantize_ex(ctypes.byref(qn), E.FP8_QUANTIZE_DEFER_RING_STEP, None) == E.FP8_ERR_INVALID_ARG
    assert f.fp8_quantize_ex(None, 0, None) == E.FP8_ERR_INVALID_ARG
    empty = fp8.QuantizeArgs(A, 0, 0, 32, 32, 0, A + 0x1000, 16, A + 0x2000, 32, None, None)
    assert f.fp8_quantize_ex(ctypes.byref(empty), E.FP8_QUANTIZE_DEFER_RING_STEP, None) == E.FP8_OK
    assert f.fp8_ring_finalize(None, 16, 0, None, None) == E.FP8_ERR_INVALID_ARG
    assert f.fp8_ring_finalize(A + 2, 16, 0, None, None) == E.FP8_ERR_INVALID_ARG
    assert f.fp8_ring_finalize(A, 0, 0, None, None) == E.FP8_ERR_INVALID_ARG
    assert f.fp8_ring_finalize(A, 16, 3, None, None) == E.FP8_ERR_INVALID_ARG


def test_mm_validation(fp8):
    E = fp8
    assert mm(fp8, scale_a=None) == E.FP8_ERR_INVALID_ARG
    assert mm(fp8, d=None) == E.FP8_ERR_INVALID_ARG
    assert mm(fp8, a_major=2) == E.FP8_ERR_INVALID_ARG
    assert mm(fp8, fmt_b=3) == E.FP8_ERR_INVALID_ARG
    assert mm(fp8, lda=136 - 4) == E.FP8_ERR_MISALIGNED
    assert mm(fp8, lda=112) == E.FP8_ERR_INVALID_ARG                  # lda < k
    assert mm(fp8, a_major=1, m=300, lda=288) == E.FP8_ERR_INVALID_ARG   # MN-major: lda >= m
    assert mm(fp8, b=A + 4) == E.FP8_ERR_MISALIGNED
    assert mm(fp8, ldd=100) == E.FP8_ERR_INVALID_ARG
    assert mm(fp8, bias=A, bias_dtype=E.FP8_DT_E4M3) == E.FP8_ERR_INVALID_ARG  # fp8 bias needs a scale
    assert mm(fp8, bias=A, bias_dtype=E.FP8_DT_FP32) == E.FP8_ERR_INVALID_ARG
    assert mm(fp8, tile_cfg=5) == E.FP8_ERR_INVALID_ARG
    assert mm(fp8, tile_cfg=-1) == E.FP8_ERR_INVALID_ARG
    assert mm(fp8, m=0) == E.FP8_OK
    assert mm(fp8, n=0, k=0) == E.FP8_OK          # empty output: nothing enqueued (K = 0 alone writes D = bias)
    assert mm(fp8, m=0, a=None, d=None) == E.FP8_OK   # empty operands and output are not dereferenced
    assert fp8._lib.fp8_mm(None, None) == E.FP8_ERR_INVALID_ARG


def test_dbias_workspace_rules(fp8):
    E = fp8
    assert fp8.fp8_dbias_workspace_bytes(0, 10) == 0
    need = fp8.fp8_dbias_workspace_bytes(2048, 1024)
    assert need > 0 and need % 16 == 0
    # fp8_dbias and the column-sum quantize (standalone or in the linear
    # backward) share one workspace size
    lin = fp8.fp8_linear_workspace_bytes(2048, 1024, 4096)
    assert lin == need
    assert fp8.fp8_linear_workspace_bytes(0, 1024, 4096) == 0
    f = fp8._lib.fp8_dbias
    assert f(A, E.FP8_DT_BF16, 2048, 1024, 1024, None, A + 0x100, None, 0, None) == E.FP8_ERR_WORKSPACE
    assert f(A, E.FP8_DT_BF16, 2048, 1024, 1024, None, A + 0x100, A, need - 16, None) == E.FP8_ERR_WORKSPACE
    assert f(A, E.FP8_DT_E5M2, 2048, 1024, 1024, None, A + 0x100, A, need, None) == E.FP8_ERR_INVALID_ARG
    assert f(A, E.FP8_DT_BF16, 2048, 1024, 1000, None, A + 0x100, A, need, None) == E.FP8_ERR_INVALID_ARG
    assert f(A, E.FP8_DT_BF16, 0, 1024, 1024, None, A + 0x100, None, 0, None) == E.FP8_OK


def fwd(fp8, **kw):
    a = dict(M=64, N=192, K=128, x=A, x_dtype=0, ldx=128, x_scale_in=None, w=A + 0x10000, w_dtype=0, ldw=128,
             w_scale_in=None, bias=None, bias_dtype=0, bias_scale=None, fmt_x=0, fmt_w=0, hist_len=16,
             ring_x=A + 0x20000, ring_w=A + 0x20100, x8=A + 0x30000, ldx8=128, w8=A + 0x40000, ldw8=128,
             sx_out=A + 0x50000, sw_out=A + 0x50010, amax_x_out=None, amax_w_out=None, y=A + 0x60000, ldy=192)
    a.update(kw)
    return fp8._lib.fp8_linear_forward(ctypes.byref(fp8.LinearFwdArgs(**a)), None)


def test_linear_forward_validation(fp8):
    E = fp8
    assert fwd(fp8, ring_w=A + 0x20000) == E.FP8_ERR_INVALID_ARG           # one ring for two tensors
    assert fwd(fp8, sx_out=None) == E.FP8_ERR_INVALID_ARG
    assert fwd(fp8, x_dtype=E.FP8_DT_E5M2, x_scale_in=A) == E.FP8_ERR_INVALID_ARG  # fmt mismatch
    assert fwd(fp8, w_dtype=E.FP8_DT_E4M3) == E.FP8_ERR_INVALID_ARG        # pre-quantized needs its scale
    assert fwd(fp8, w_dtype=E.FP8_DT_E4M3, w_scale_in=A, ldw=136) == E.FP8_ERR_MISALIGNED
    assert fwd(fp8, ldx8=136) == E.FP8_ERR_MISALIGNED
    assert fwd(fp8, ldx8=120) == E.FP8_ERR_INVALID_ARG
    assert fwd(fp8, ldy=100) == E.FP8_ERR_INVALID_ARG
    assert fwd(fp8, hist_len=0) == E.FP8_ERR_INVALID_ARG
    assert fwd(fp8, M=0, N=0) == E.FP8_OK       # x and w empty: nothing enqueued
    assert fwd(fp8, M=0, N=0, x=None, w=None) == E.FP8_OK
    assert fp8._lib.fp8_linear_forward(None, None) == E.FP8_ERR_INVALID_ARG


def bwd(fp8, **kw):
    a = dict(M=64, N=192, K=128, g=A, g_dtype=0, ldg=192, g_scale_in=None, fmt_g=1, hist_len=16,
             ring_g=A + 0x20000, g8=A + 0x30000, ldg8=192, sg_out=A + 0x50000, amax_g_out=None,
             x8=A + 0x40000, ldx8=128, sx=A + 0x50010, fmt_x=0, w8=A + 0x70000, ldw8=128, sw=A + 0x50020, fmt_w=0,
             need_dx=1, need_dw=1, need_dbias=0, dx=A + 0x80000, lddx=128, dw=A + 0x90000, lddw=128, dbias=None,
             workspace=None, workspace_bytes=0)
    a.update(kw)
    return fp8._lib.fp8_linear_backward(ctypes.byref(fp8.LinearBwdArgs(**a)), None)


def test_linear_backward_validation(fp8):
    E = fp8
    assert bwd(fp8, need_dbias=1, dbias=A) == E.FP8_ERR_WORKSPACE
    assert bwd(fp8, need_dbias=1, dbias=None) == E.FP8_ERR_INVALID_ARG
    assert bwd(fp8, sw=None) == E.FP8_ERR_INVALID_ARG
    assert bwd(fp8, ldw8=136) == E.FP8_ERR_MISALIGNED
    assert bwd(fp8, ldx8=136, need_dw=1) == E.FP8_ERR_MISALIGNED
    assert bwd(fp8, g_dtype=E.FP8_DT_E5M2) == E.FP8_ERR_INVALID_ARG         # pre-quantized g needs its scale
    assert bwd(fp8, sg_out=None) == E.FP8_ERR_INVALID_ARG
    assert bwd(fp8, N=0, need_dx=0) == E.FP8_OK  # g and dW empty: nothing enqueued
    assert bwd(fp8, M=0, need_dw=0, g=None) == E.FP8_OK
    # one workspace size serves fp8_dbias, fp8_quantize_dbias and the
    # backward's column sums; one byte short of it is refused
    M, N, K = 2048, 1024, 1024
    lin, dbw = fp8.fp8_linear_workspace_bytes(M, N, K), fp8.fp8_dbias_workspace_bytes(M, N)
    assert lin == dbw
    big = dict(M=M, N=N, K=K, ldg=N, ldg8=N, ldx8=K, ldw8=K, lddx=K, lddw=K, need_dbias=1, dbias=A + 0xA0000,
               workspace=A + 0x100000)
    assert bwd(fp8, workspace_bytes=lin - 1, **big) == E.FP8_ERR_WORKSPACE
    assert bwd(fp8, workspace_bytes=lin, workspace=A + 0x100008, **{k: v for k, v in big.items()
                                                                   if k != "workspace"}) == E.FP8_ERR_WORKSPACE


def test_colsum_split_stays_in_one_wave(fp8):
    # the column-sum quantize runs at most 444 blocks (three per SM on 148
    # SMs): 43 column tiles of 11008 columns get 10 row splits, not 11 (473
    # blocks would spill into a second wave); 27 tiles of 6912 get 16, not 17
    for M, N, tiles, R in ((4096, 11008, 43, 10), (2048, 6912, 27, 16), (4096, 4096, 16, 27)):
        counters = (tiles * 4 + 15) // 16 * 16
        assert fp8.fp8_dbias_workspace_bytes(M, N) == counters + R * N * 4, (M, N)


def test_bias_gradient_split_bounds(fp8):
    # for any shape, the row splits R behind the workspace size keep every
    # column-sum grid (col tiles x R) within one wave of 444 blocks unless a
    # single split per tile already exceeds it, and never split below 32 rows
    for M in (1, 31, 32, 33, 100, 512, 2048, 3000, 4096, 65536):
        for N in (1, 255, 256, 257, 1024, 6912, 11008, 120000):
            tiles = -(-N // 256)
            counters = (tiles * 4 + 15) // 16 * 16
            part = fp8.fp8_dbias_workspace_bytes(M, N) - counters   # R x N fp32, 16-byte rounded
            r16 = lambda r: (r * N * 4 + 15) // 16 * 16  # noqa: E731
            bound = min(max(1, 444 // tiles), -(-M // 32))
            assert r16(1) <= part <= r16(bound), (M, N, part, bound)


def test_linear_workspace_covers_dbias(fp8):
    for M in (1, 3, 64, 100, 512, 2048, 4096, 65536):
        for N in (1, 100, 192, 1024, 1536, 4096, 6912, 11008):
            lin, dbw = fp8.fp8_linear_workspace_bytes(M, N, 64), fp8.fp8_dbias_workspace_bytes(M, N)
            assert lin == dbw > 0 and lin % 16 == 0


def test_fused_entry_points_validation(fp8):
    E = fp8
    qa = fp8.QuantizeArgs(A, 0, 4, 32, 32, 0, A + 0x1000, 16, A + 0x2000, 32, None, None)
    qb = fp8.QuantizeArgs(A + 0x3000, 0, 8, 32, 32, 0, A + 0x4000, 16, A + 0x5000, 32, None, None)
    same_ring = fp8.QuantizeArgs(A + 0x3000, 0, 8, 32, 32, 0, A + 0x1000, 16, A + 0x5000, 32, None, None)
    other_fmt = fp8.QuantizeArgs(A + 0x3000, 0, 8, 32, 32, 1, A + 0x4000, 16, A + 0x5000, 32, None, None)
    f = fp8._lib
    assert f.fp8_quantize_dual(ctypes.byref(qa), ctypes.byref(same_ring), None) == E.FP8_ERR_INVALID_ARG
    assert f.fp8_quantize_dual(ctypes.byref(qa), ctypes.byref(other_fmt), None) == E.FP8_ERR_INVALID_ARG
    assert f.fp8_quantize_dual(None, ctypes.byref(qb), None) == E.FP8_ERR_INVALID_ARG
    empty = fp8.QuantizeArgs(A, 0, 0, 32, 32, 0, A + 0x1000, 16, A + 0x2000, 32, None, None)
    empty2 = fp8.QuantizeArgs(A, 0, 0, 32, 32, 0, A + 0x4000, 16, A + 0x2000, 32, None, None)
    assert f.fp8_quantize_dual(ctypes.byref(empty), ctypes.byref(empty2), None) == E.FP8_OK
    assert f.fp8_quantize_dbias(ctypes.byref(qa), A + 0x9000, None, 0, None) == E.FP8_ERR_WORKSPACE
    assert f.fp8_quantize_dbias(ctypes.byref(qa), None, A, 1 << 20, None) == E.FP8_ERR_INVALID_ARG
    assert f.fp8_quantize_dbias(ctypes.byref(empty), A + 0x9000, None, 0, None) == E.FP8_OK
    good = fp8.MmArgs(m=128, n=128, k=128, a=A, lda=128, b=A + 0x10000, ldb=128, scale_a=A + 0x20000,
                      scale_b=A + 0x20010, d=A + 0x30000, ldd=128)
    bad = fp8.MmArgs(m=128, n=128, k=128, a=A, lda=120, b=A + 0x10000, ldb=128, scale_a=A + 0x20000,
                     scale_b=A + 0x20010, d=A + 0x30000, ldd=128)
    assert f.fp8_mm_pair(ctypes.byref(good), ctypes.byref(bad), None) == E.FP8_ERR_INVALID_ARG
    assert f.fp8_mm_pair(None, ctypes.byref(good), None) == E.FP8_ERR_INVALID_ARG
    zero = fp8.MmArgs(m=0, n=128, k=128, a=A, lda=128, b=A + 0x10000, ldb=128, scale_a=A + 0x20000,
                      scale_b=A + 0x20010, d=A + 0x30000, ldd=128)
    assert f.fp8_mm_pair(ctypes.byref(zero), ctypes.byref(zero), None) == E.FP8_OK


def test_wait_selftest_validation(fp8):
    """Arguments are checked before anything is launched (no GPU needed)."""
    f = fp8._lib.fp8_wait_selftest
    assert f(None, 1000, 0x1000, None) == fp8.FP8_ERR_INVALID_ARG
    assert f(0x1000, 1000, None, None) == fp8.FP8_ERR_INVALID_ARG
    assert f(0x1002, 1000, 0x1000, None) == fp8.FP8_ERR_INVALID_ARG     # flag not 4-byte aligned
    assert f(0x1000, 1000, 0x1001, None) == fp8.FP8_ERR_INVALID_ARG     # results not 4-byte aligned
    assert f(0x1000, 0, 0x1000, None) == fp8.FP8_ERR_INVALID_ARG        # no limit
    assert f(0x1000, 2_000_000_001, 0x1000, None) == fp8.FP8_ERR_INVALID_ARG  # above 2 s
