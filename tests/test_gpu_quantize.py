"""GPU parity of the quantize + in-kernel ring finalize against the oracle.
fp8 codes, amax, the scale snapshot and every ring word must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import (assert_codes_equal, bits, dt_code, fp8_buffer, host_rows, oracle_ring_words, padded,
                     ring_words)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def gpu_quantize(fp8, x_dev, fmt, ring, ld_out=None):
    rows, cols = x_dev.shape
    out = fp8_buffer(rows, cols, ld_out)
    amax = torch.full((1,), -1.0, device="cuda")
    scale = torch.full((1,), -1.0, device="cuda")
    fp8.fp8_quantize(x_dev, fmt, ring.buf, ring.H, out, amax, scale)
    torch.cuda.synchronize()
    return out, amax.item(), scale.item()


def check_step(fp8, x_cpu, fmt, ring, oring, ld_in=None, ld_out=None):
    rows, cols = x_cpu.shape
    x_dev = padded(x_cpu, ld_in) if ld_in else x_cpu.cuda()
    out, amax, scale = gpu_quantize(fp8, x_dev, fmt, ring, ld_out)
    xb = bits(x_cpu)
    q, a, s = oracle.quantize(xb, dt_code(x_cpu), fmt, oring)
    assert np.float32(scale) == s, (scale, s)
    assert np.float32(amax).view(np.uint32) == np.float32(a).view(np.uint32), (amax, a)
    assert_codes_equal(host_rows(out), q, fmt)
    ldo = out.stride(0)
    if ldo > cols:
        base = torch.as_strided(out, (rows, ldo), (ldo, 1))
        pad = base[:, cols:].cpu()
        assert bool((pad == 0).all()), "padding bytes must be written as zero"
    assert np.array_equal(ring_words(ring), oracle_ring_words(oring)), (ring_words(ring), oracle_ring_words(oring))
    return out


def test_ring_evolution_c1(fp8):
    """Config 1: x ~ N(0,1) 2^step, 4 delayed steps, H=16: codes, amax,
    snapshot and ring words bit-exact at every step (the doubling amax makes
    the delayed scale saturate the top values)."""
    ring = fp8.ScaleRing(wl.HIST_LEN)
    oring = oracle.Ring(wl.HIST_LEN)
    M, K = wl.C1.M, wl.C1.K
    for step in range(wl.C1_STEPS):
        x = wl.normal((M, K), 2.0 ** step, wl.seed_for(1, step, wl.OP_X))
        check_step(fp8, x, fp8.FP8_E4M3, ring, oring)
    assert ring.step == wl.C1_STEPS


@pytest.mark.parametrize("dtype", (torch.bfloat16, torch.float16, torch.float32))
@pytest.mark.parametrize("fmt", (0, 1))
@pytest.mark.parametrize("rows,cols,ld_in,ld_out", [
    (37, 53, 61, 64), (1, 7, 7, 16), (2048, 7, 7, 16), (3, 1534, 1534, 1536), (300, 100, 104, 112),
    (64, 128, 128, 128), (2048, 1024, 1024, 1024), (513, 4096, 4100, 4096)])
def test_quantize_shapes(fp8, dtype, fmt, rows, cols, ld_in, ld_out):
    """Ragged, strided, single-row, odd-K and contiguous tensors, three steps
    each so the history and step counter move."""
    ring = fp8.ScaleRing(16)
    oring = oracle.Ring(16)
    for step in range(3):
        std = (1.0, 37.0, 0.01)[step] * (1000.0 if fmt == 1 else 1.0)
        x = wl.normal((rows, cols), std, 777 + step + rows, dtype=dtype)
        check_step(fp8, x, fmt, ring, oring, ld_in=ld_in if ld_in != cols else None, ld_out=ld_out)


def test_quantize_special_values(fp8):
    """NaN (ignored by amax, NaN code), +-inf (saturate; amax inf keeps the old
    scale), -0, values that round to zero, exact ties after scaling."""
    vals = np.array([np.nan, np.inf, -np.inf, -0.0, 0.0, 1e-30, -1e-30, 448.0, 449.0, 464.0, 1e6, -1e6,
                     3.0, 0.5, 2.0 ** -10, 2.0 ** -9, 1.0625, 1.1875], np.float32)
    x = torch.from_numpy(np.tile(vals, (5, 3)).astype(np.float32))
    for fmt in (0, 1):
        ring = fp8.ScaleRing(4)
        oring = oracle.Ring(4)
        check_step(fp8, x, fmt, ring, oring)           # amax inf -> scale kept at 1
        check_step(fp8, x.to(torch.bfloat16), fmt, ring, oring)
        xf = torch.nan_to_num(x, posinf=3.0e4, neginf=-2.0e4)
        check_step(fp8, xf, fmt, ring, oring)
        check_step(fp8, x, fmt, ring, oring)


def test_quantize_large_many_blocks(fp8):
    """c4 x with 0.1% outliers x50 (4096 x 4096) and c3 x (2048 x 6912): a grid
    of hundreds of blocks, bit-exact codes and ring."""
    ring = fp8.ScaleRing(16)
    oring = oracle.Ring(16)
    x = wl.normal_with_outliers((4096, 4096), 1.0, wl.seed_for(4, 0, wl.OP_X), wl.seed_for(4, 0, wl.OP_MASK))
    check_step(fp8, x, 0, ring, oring)
    x2 = wl.normal((2048, 6912), 1.0, wl.seed_for(3, 0, wl.OP_X))
    check_step(fp8, x2, 0, ring, oring)
    check_step(fp8, x, 0, ring, oring)


def test_ring_init_seed(fp8):
    for fmt, amax in ((0, 3.5), (1, 1e-3), (0, 0.0), (0, float("inf")), (1, 1e-42)):
        ring = fp8.ScaleRing(16, seed_amax=amax, fmt=fmt)
        oring = oracle.Ring(16)
        oring.seed(amax, fmt)
        torch.cuda.synchronize()
        assert np.array_equal(ring_words(ring), oracle_ring_words(oring)), (fmt, amax)


def test_ring_checkpoint_resume(fp8):
    """Copying a ring's bytes between launches checkpoints it: resuming from the
    copy gives the same scales as the uninterrupted run."""
    ring = fp8.ScaleRing(8)
    xs = [wl.normal((256, 256), 1.5 ** i, 4242 + i).cuda() for i in range(12)]
    out = fp8_buffer(256, 256)
    for x in xs[:5]:
        fp8.fp8_quantize(x, 0, ring.buf, 8, out)
    saved = ring.buf.clone()
    for x in xs[5:]:
        fp8.fp8_quantize(x, 0, ring.buf, 8, out)
    ring.buf.copy_(saved)
    for x in xs[5:]:
        fp8.fp8_quantize(x, 0, ring.buf, 8, out)
    a = ring.buf.clone()
    ring2 = fp8.ScaleRing(8)
    for x in xs:
        fp8.fp8_quantize(x, 0, ring2.buf, 8, out)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), ring2.buf.view(torch.int32))


def test_no_device_timeouts_recorded(fp8):
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0


@pytest.mark.parametrize("dtype", (torch.bfloat16, torch.float32))
def test_quantize_dual_matches_two_launches(fp8, dtype):
    """fp8_quantize_dual on (x, w) = two fp8_quantize calls: same codes, amax,
    snapshots and ring words, for several steps."""
    H = 16
    r1, r2 = fp8.ScaleRing(H), fp8.ScaleRing(H)
    o1, o2 = oracle.Ring(H), oracle.Ring(H)
    for step in range(3):
        x = wl.normal((2048, 1024), 1.0 + step, 900 + step, dtype=dtype)
        w = wl.normal((1000, 1024), 0.03 * (3 - step), 950 + step, dtype=dtype)
        xd, wd = x.cuda(), w.cuda()
        x8, w8 = fp8_buffer(2048, 1024), fp8_buffer(1000, 1024)
        sc = torch.zeros(4, device="cuda")
        a = fp8.quantize_args(xd, 0, r1.buf, H, x8, sc[0:1], sc[1:2])
        b = fp8.quantize_args(wd, 0, r2.buf, H, w8, sc[2:3], sc[3:4])
        fp8.fp8_quantize_dual(a, b)
        torch.cuda.synchronize()
        qx, ax, sx = oracle.quantize(bits(x), dt_code(x), 0, o1)
        qw, aw, sw = oracle.quantize(bits(w), dt_code(w), 0, o2)
        assert sc.tolist() == [ax, sx, aw, sw]
        assert_codes_equal(host_rows(x8), qx, 0)
        assert_codes_equal(host_rows(w8), qw, 0)
        assert np.array_equal(ring_words(r1), oracle_ring_words(o1))
        assert np.array_equal(ring_words(r2), oracle_ring_words(o2))


@pytest.mark.parametrize("rows,cols", [(2048, 1024), (300, 100), (4096, 4096), (1, 7), (77, 1534), (3, 120000),
                                       (300, 113920)])
def test_quantize_dbias_entry(fp8, rows, cols):
    """fp8_quantize_dbias: codes and ring bit-exact, dbias within
    max(1 bf16 ulp, 2e-6 sum|g|) of the oracle's column sums."""
    H = 16
    ring = fp8.ScaleRing(H)
    orr = oracle.Ring(H)
    ws = torch.zeros(max(16, fp8.fp8_dbias_workspace_bytes(rows, cols)), dtype=torch.uint8, device="cuda")
    for step in range(2):
        g = wl.normal((rows, cols), 1e-3 * (1 + 3 * step), 970 + step)
        out = fp8_buffer(rows, cols)
        db = torch.empty(cols, dtype=torch.bfloat16, device="cuda")
        gd = g.cuda()  # the args hold a raw pointer: keep the tensor alive
        fp8.fp8_quantize_dbias(fp8.quantize_args(gd, 1, ring.buf, H, out), db, ws)
        torch.cuda.synchronize()
        q, a, s = oracle.quantize(bits(g), oracle.DT_BF16, 1, orr)
        assert_codes_equal(host_rows(out), q, 1)
        assert np.array_equal(ring_words(ring), oracle_ring_words(orr))
        want, _, sa = oracle.dbias(bits(g), oracle.DT_BF16, rows, cols)
        gv = oracle.bf16_to_f32(bits(db.cpu())).astype(np.float64)
        ov = oracle.bf16_to_f32(want).astype(np.float64)
        assert np.all(np.abs(gv - ov) <= np.maximum(oracle.bf16_ulp(ov), 2e-6 * sa))
    assert fp8.fp8_get_device_status() == 0


def dbias_close(db, want, sa, what):
    gv = oracle.bf16_to_f32(bits(db.cpu())).astype(np.float64)
    ov = oracle.bf16_to_f32(want).astype(np.float64)
    assert np.all(np.abs(gv - ov) <= np.maximum(oracle.bf16_ulp(ov), 2e-6 * sa)), what


@pytest.mark.parametrize("rows,cols", [(2048, 1024), (77, 1534), (1, 300), (1000, 11008), (3, 120000),
                                       (300, 113920)])
def test_dbias_entry(fp8, rows, cols):
    """fp8_dbias against the oracle's column sums, within max(1 bf16 ulp,
    2e-6 sum|g|): bf16 and fp32 g, and E4M3 codes with a scale (dequantized
    before the sum); shapes from one row split to many, and with more than
    444 column tiles (one split per tile), each call twice on one workspace
    (the tile counters back at zero between calls)."""
    ws = torch.zeros(max(16, fp8.fp8_dbias_workspace_bytes(rows, cols)), dtype=torch.uint8, device="cuda")
    for dtype in (torch.bfloat16, torch.float32):
        g = wl.normal((rows, cols), 1e-3, 990 + rows, dtype=dtype)
        gd = g.cuda()
        want, _, sa = oracle.dbias(bits(g) if dtype == torch.bfloat16 else g.numpy().view(np.uint32),
                                   dt_code(g), rows, cols)
        for _ in range(2):
            db = torch.empty(cols, dtype=torch.bfloat16, device="cuda")
            fp8.fp8_dbias(gd, db, ws)
            torch.cuda.synchronize()
            dbias_close(db, want, sa, (rows, cols, dtype))
    gen = torch.Generator().manual_seed(rows + cols)
    codes = (torch.randint(0, 0x7E, (rows, cols), generator=gen, dtype=torch.int32) |
             (torch.randint(0, 2, (rows, cols), generator=gen, dtype=torch.int32) << 7)).to(torch.uint8)  # no NaN
    sg = torch.tensor([19.25], device="cuda")
    db = torch.empty(cols, dtype=torch.bfloat16, device="cuda")
    fp8.fp8_dbias(codes.cuda(), db, ws, g_scale=sg, g_fmt=fp8.FP8_E4M3)
    torch.cuda.synchronize()
    want, _, sa = oracle.dbias(codes.numpy(), oracle.DT_E4M3, rows, cols, 19.25)
    dbias_close(db, want, sa, (rows, cols, "e4m3"))
    assert fp8.fp8_get_device_status() == 0


@pytest.mark.parametrize("H,offset", [(1, 0), (3, 0), (5, 0), (16, 4), (6, 4), (16, 0), (2, 0)])
def test_ring_finalize_paths(fp8, H, offset):
    """Both forms of the last-block finalize against the oracle over several
    multi-block steps: with an even H and an 8-byte aligned ring, ticket and
    scratch share one 8-byte word (one 64-bit atomic per block); an odd H or a
    ring only 4-byte aligned (offset 4 bytes) takes the two-word protocol.
    Codes, amax, snapshot and every ring word bit for bit; also through the
    column-sum quantize (fp8_quantize_dbias) and the dual launch."""
    words = fp8.fp8_ring_bytes(H) // 4
    k = offset // 4

    def ring_at(tag):
        base = torch.zeros(words + 2, dtype=torch.float32, device="cuda")
        r = fp8.ScaleRing(H, buf=base[k:k + words])
        fp8.fp8_ring_init(r.buf, H)
        assert (r.buf.data_ptr() % 8 == 0) == (offset == 0)
        return r

    ring, oring = ring_at(0), oracle.Ring(H)
    for step in range(H + 3):  # wraps the history at least once
        x = wl.normal((1536, 1000), 0.5 * (1.3 ** (step % 7)), 7100 + step)
        check_step(fp8, x, fp8.FP8_E4M3 if step % 2 == 0 else fp8.FP8_E5M2, ring, oring)
    # column-sum quantize (the bias-gradient path) on the same kind of ring
    rg, org = ring_at(1), oracle.Ring(H)
    rows, cols = 700, 600
    ws = torch.zeros(max(16, fp8.fp8_dbias_workspace_bytes(rows, cols)), dtype=torch.uint8, device="cuda")
    for step in range(3):
        g = wl.normal((rows, cols), 1e-3 * (1 + step), 7200 + step)
        gd, out = g.cuda(), fp8_buffer(rows, cols)
        db = torch.empty(cols, dtype=torch.bfloat16, device="cuda")
        fp8.fp8_quantize_dbias(fp8.quantize_args(gd, 1, rg.buf, H, out), db, ws)
        torch.cuda.synchronize()
        q, _, _ = oracle.quantize(bits(g), oracle.DT_BF16, 1, org)
        assert_codes_equal(host_rows(out), q, 1)
        assert np.array_equal(ring_words(rg), oracle_ring_words(org))
    # dual launch: two rings of this kind in one grid
    r1, r2, o1, o2 = ring_at(2), ring_at(3), oracle.Ring(H), oracle.Ring(H)
    for step in range(3):
        x = wl.normal((1024, 640), 1.0 + step, 7300 + step)
        w = wl.normal((512, 640), 0.05, 7350 + step)
        xd, wd = x.cuda(), w.cuda()
        x8, w8 = fp8_buffer(1024, 640), fp8_buffer(512, 640)
        fp8.fp8_quantize_dual(fp8.quantize_args(xd, 0, r1.buf, H, x8), fp8.quantize_args(wd, 0, r2.buf, H, w8))
        torch.cuda.synchronize()
        oracle.quantize(bits(x), dt_code(x), 0, o1)
        oracle.quantize(bits(w), dt_code(w), 0, o2)
        assert np.array_equal(ring_words(r1), oracle_ring_words(o1))
        assert np.array_equal(ring_words(r2), oracle_ring_words(o2))
    assert fp8.fp8_get_device_status() == 0
