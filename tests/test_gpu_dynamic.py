"""GPU parity of current (dynamic) scaling -- ring NULL, the scale taken from
the tensor's own amax -- against the oracle: codes, amax and scale bit for bit,
GEMMs within max(1 bf16 ulp, 2e-6 sum|ab| / (sa sb)), for fp8_quantize, the
dual and column-sum entry points, and the fused linear forward/backward."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import assert_codes_equal, bits, dt_code, fp8_buffer, host_rows, oracle_ring_words, padded, ring_words
from test_gpu_linear import dbias_check, gemm_check

pytestmark = pytest.mark.gpu
E4, E5 = oracle.E4M3, oracle.E5M2


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def dyn_check(fp8, x_cpu, fmt, ld_in=None, ld_out=None):
    rows, cols = x_cpu.shape
    x_dev = padded(x_cpu, ld_in) if ld_in else x_cpu.cuda()
    out = fp8_buffer(rows, cols, ld_out)
    amax = torch.full((1,), -1.0, device="cuda")
    scale = torch.full((1,), -1.0, device="cuda")
    fp8.fp8_quantize(x_dev, fmt, None, 0, out, amax, scale)
    torch.cuda.synchronize()
    q, a, s = oracle.quantize_dynamic(bits(x_cpu), dt_code(x_cpu), fmt)
    assert np.float32(amax.item()).view(np.uint32) == np.float32(a).view(np.uint32), (amax.item(), a)
    assert np.float32(scale.item()) == s, (scale.item(), s)
    assert_codes_equal(host_rows(out), q, fmt)
    return out


@pytest.mark.parametrize("dtype", (torch.bfloat16, torch.float16, torch.float32))
@pytest.mark.parametrize("fmt", (0, 1))
@pytest.mark.parametrize("rows,cols,ld_in,ld_out", [
    (37, 53, 61, 64), (1, 7, 7, 16), (300, 100, 104, 112), (2048, 1024, 1024, 1024), (513, 4096, 4100, 4096)])
def test_quantize_dynamic_shapes(fp8, dtype, fmt, rows, cols, ld_in, ld_out):
    for i, std in enumerate((1.0, 3e3, 1e-3)):
        x = wl.normal((rows, cols), std, 1200 + i + rows, dtype=dtype)
        dyn_check(fp8, x, fmt, ld_in=ld_in if ld_in != cols else None, ld_out=ld_out)


def test_quantize_dynamic_specials_and_repeat(fp8):
    """All zeros (scale 1, amax 0), NaN and inf (amax inf -> scale 1), and the
    same tensor twice (the amax word is cleared before each reduction)."""
    z = torch.zeros((64, 96), dtype=torch.bfloat16)
    dyn_check(fp8, z, 0)
    x = wl.normal((64, 96), 2.0, 1300)
    x[3, 5] = float("nan")
    dyn_check(fp8, x, 0)
    x[7, 9] = float("inf")
    dyn_check(fp8, x, 1)
    y = wl.normal((500, 300), 0.5, 1301)
    dyn_check(fp8, y, 0)
    dyn_check(fp8, y, 0)


def test_dual_dynamic_and_delayed(fp8):
    """fp8_quantize_dual with x on current scaling and w on a ring, then both
    on current scaling: same bytes as the oracle's separate paths."""
    H = 16
    rw, orw = fp8.ScaleRing(H), oracle.Ring(H)
    for step in range(2):
        x = wl.normal((2048, 1024), 1.0 + 5 * step, 1400 + step)
        w = wl.normal((1000, 1024), 0.03, 1450 + step)
        x8, w8 = fp8_buffer(2048, 1024), fp8_buffer(1000, 1024)
        sc = torch.zeros(4, device="cuda")
        xd, wd = x.cuda(), w.cuda()  # the args hold raw pointers: keep the tensors alive
        a = fp8.quantize_args(xd, 0, None, 0, x8, sc[0:1], sc[1:2])
        b = fp8.quantize_args(wd, 0, rw.buf, H, w8, sc[2:3], sc[3:4])
        fp8.fp8_quantize_dual(a, b)
        torch.cuda.synchronize()
        qx, ax, sx = oracle.quantize_dynamic(bits(x), oracle.DT_BF16, 0)
        qw, aw, sw = oracle.quantize(bits(w), oracle.DT_BF16, 0, orw)
        assert sc.tolist() == [ax, sx, aw, sw]
        assert_codes_equal(host_rows(x8), qx, 0)
        assert_codes_equal(host_rows(w8), qw, 0)
        assert np.array_equal(ring_words(rw), oracle_ring_words(orw))
    # both dynamic
    x = wl.normal((700, 520), 9.0, 1460)
    w = wl.normal((520, 520), 0.1, 1461)
    x8, w8 = fp8_buffer(700, 520), fp8_buffer(520, 520)
    # -1.0 (0xBF800000) is above every finite |x| as raw bits: both amax words
    # must be cleared before the reduction, or they keep it
    sc = torch.full((4,), -1.0, device="cuda")
    xd, wd = x.cuda(), w.cuda()
    fp8.fp8_quantize_dual(fp8.quantize_args(xd, 1, None, 0, x8, sc[0:1], sc[1:2]),
                          fp8.quantize_args(wd, 1, None, 0, w8, sc[2:3], sc[3:4]))
    torch.cuda.synchronize()
    qx, ax, sx = oracle.quantize_dynamic(bits(x), oracle.DT_BF16, 1)
    qw, aw, sw = oracle.quantize_dynamic(bits(w), oracle.DT_BF16, 1)
    assert sc.tolist() == [ax, sx, aw, sw]
    assert_codes_equal(host_rows(x8), qx, 1)
    assert_codes_equal(host_rows(w8), qw, 1)


@pytest.mark.parametrize("rows,cols", [(2048, 1024), (300, 100), (77, 1534)])
def test_quantize_dbias_dynamic(fp8, rows, cols):
    ws = torch.zeros(max(16, fp8.fp8_dbias_workspace_bytes(rows, cols)), dtype=torch.uint8, device="cuda")
    g = wl.normal((rows, cols), 1e-3, 1500 + rows)
    out = fp8_buffer(rows, cols)
    db = torch.empty(cols, dtype=torch.bfloat16, device="cuda")
    sc = torch.zeros(2, device="cuda")
    gd = g.cuda()
    fp8.fp8_quantize_dbias(fp8.quantize_args(gd, 1, None, 0, out, sc[0:1], sc[1:2]), db, ws)
    torch.cuda.synchronize()
    q, a, s = oracle.quantize_dynamic(bits(g), oracle.DT_BF16, 1)
    assert sc.tolist() == [a, s]
    assert_codes_equal(host_rows(out), q, 1)
    dbias_check(db, bits(g), rows, cols)


@pytest.mark.parametrize("shape,full", [(wl.C1, True), (wl.C2_LAYER[4], False)], ids=["c1", "c2_up"])
def test_linear_dynamic(fp8, shape, full):
    """fp8_linear_forward/backward with all rings NULL: every operand scaled by
    its own amax; the backward still reuses the forward's scales."""
    M, K, N = shape.M, shape.K, shape.N
    rng = np.random.default_rng(15)
    for step in range(2):
        x = wl.normal((M, K), 2.0 ** (4 * step), 1600 + step)
        w = wl.normal((N, K), wl.weight_std(K), 1610 + step)
        g = wl.normal((M, N), 1e-3, 1620 + step)
        bias = wl.normal((N,), 0.01, 1630)
        f = fp8.linear_forward(x.cuda(), w.cuda(), None, None, bias=bias.cuda())
        b = fp8.linear_backward(g.cuda(), f, None, need_dbias=True)
        torch.cuda.synchronize()
        assert fp8.fp8_get_device_status() == 0
        fo = oracle.linear_forward(M, N, K, bits(x), oracle.DT_BF16, bits(w), oracle.DT_BF16, None, None,
                                   bias=bits(bias), ldx8=(K + 15) // 16 * 16, ldw8=(K + 15) // 16 * 16, sumabs=False)
        g8o, ag, sg = oracle.quantize_dynamic(bits(g), oracle.DT_BF16, E5, ld_out=(N + 15) // 16 * 16)
        assert (f.sx.item(), f.sw.item(), b.sg.item()) == (fo["sx"], fo["sw"], sg)
        assert (f.amax_x.item(), f.amax_w.item(), b.amax_g.item()) == (fo["amax_x"], fo["amax_w"], ag)
        x8o, w8o = fo["x8"], fo["w8"]
        assert_codes_equal(host_rows(f.x8), x8o[:, :K], E4)
        assert_codes_equal(host_rows(f.w8), w8o[:, :K], E4)
        assert_codes_equal(host_rows(b.g8), g8o[:, :N], E5)
        gemm_check(f.y, x8o, 0, E4, w8o, E4, M, N, K, fo["sx"], fo["sw"], "fwd", full, rng, bits(bias),
                   oracle.DT_BF16, 1.0, "dyn y")
        gemm_check(b.dx, g8o, 0, E5, w8o, E4, M, K, N, sg, fo["sw"], "dx", full, rng, what="dyn dx")
        gemm_check(b.dw, g8o, 0, E5, x8o, E4, N, K, M, sg, fo["sx"], "dw", full, rng, what="dyn dw")
        dbias_check(b.dbias, bits(g), M, N)
