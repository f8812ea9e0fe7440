"""GPU parity of the whole FP8 linear (fp8_linear_forward / fp8_linear_backward)
against the oracle's forward/backward orchestration, on the five workload
configurations: quantized operands, amaxes, scale snapshots and ring words
bit-exact; y, dX, dW within max(1 bf16 ulp, 2e-6 sum|ab| / (sa sb)); dbias
within max(1 bf16 ulp, 2e-6 sum|g|).  Large shapes compare sampled GEMM
outputs (full rows, full columns, random points); quantize is always full."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import assert_codes_equal, assert_gemm_close, bits, host_rows, oracle_ring_words, ring_words, \
    sample_points

pytestmark = pytest.mark.gpu
E4, E5 = oracle.E4M3, oracle.E5M2


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def gemm_check(y_gpu, a8, a_major_rows, fmt_a, b8, fmt_b, I, J, Kc, sa, sb, kind, full, rng, bias=None,
               bias_dtype=0, bias_scale=1.0, what=""):
    """kind: 'fwd' (A=X8 [I,Kc], B=W8 [J,Kc]), 'dx' (A=G8 [I,Kc], B=W8 [Kc,J]),
    'dw' (A=G8 [Kc,I], B=X8 [Kc,J]).  Operands are contiguous numpy arrays."""
    lda, ldb = a8.shape[1], b8.shape[1]
    a_s = {"fwd": (lda, 1), "dx": (lda, 1), "dw": (1, lda)}[kind]
    b_s = {"fwd": (ldb, 1), "dx": (1, ldb), "dw": (1, ldb)}[kind]
    y = y_gpu.cpu().view(torch.int16).numpy().view(np.uint16)
    if full:
        acc, _, sab = oracle.gemm_acc(a8, fmt_a, *a_s, b8, fmt_b, *b_s, I, J, Kc)
        want, _ = oracle.epilogue(acc, sa, sb, bias, bias_dtype, bias_scale)
        return assert_gemm_close(y, want, sab, sa, sb, what)
    pi, pj = sample_points(rng, I, J)
    acc, sab = oracle.gemm_acc_points(pi, pj, a8, fmt_a, *a_s, b8, fmt_b, *b_s, Kc)
    want, _ = oracle.epilogue(acc, sa, sb, bias, bias_dtype, bias_scale, col_idx=pj)
    return assert_gemm_close(y[pi, pj], want, sab, sa, sb, what + " (sampled)")


def dbias_check(got, g_bits, M, N):
    want, _, sa = oracle.dbias(g_bits, oracle.DT_BF16, M, N)
    g = oracle.bf16_to_f32(got.cpu().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    o = oracle.bf16_to_f32(want).astype(np.float64)
    tol = np.maximum(oracle.bf16_ulp(o), 2e-6 * sa)
    both_nan = np.isnan(g) & np.isnan(o)
    err = np.where(both_nan, 0.0, np.abs(g - o))
    assert np.all((err <= tol) | both_nan), np.nanmax(err / tol)


def prequantized_device(codes_np, scale, rows, cols):
    """fp8 codes (numpy [rows, >= cols]) in a 16-aligned device buffer, and the
    scale as a 1-element device tensor."""
    buf = torch.zeros((rows, (cols + 15) // 16 * 16), dtype=torch.uint8)
    buf[:, :cols] = torch.from_numpy(np.ascontiguousarray(codes_np[:, :cols]))
    return buf.cuda()[:, :cols], torch.tensor([scale], dtype=torch.float32, device="cuda")


def linear_step(fp8, x, w, g, rings, orings, full, rng, bias=None, bias8=None, bias_scale=None,
                need_dbias=False, w_pre=None, x_pre=None, what=""):
    """One forward + backward on the GPU and in the oracle; compare everything.
    w_pre / x_pre: (codes [N,K] / [M,K] numpy, scale) for a pre-quantized
    weight / activation: its quantize is skipped, its snapshot is the given
    scale, its amax output 0 and its ring untouched."""
    M, K = x.shape if x is not None else x_pre[0].shape
    N = w.shape[0] if w is not None else w_pre[0].shape[0]
    rx, rw, rg = rings
    orx, orw, org = orings
    dev_bias, bias_np, bias_dt, bsc = None, None, oracle.DT_BF16, 1.0
    dev_bsc = None
    if bias is not None:
        dev_bias, bias_np = bias.cuda(), bits(bias)
    elif bias8 is not None:
        dev_bias, bias_np, bias_dt, bsc = torch.from_numpy(bias8).cuda(), bias8, oracle.DT_E4M3, bias_scale
        dev_bsc = torch.tensor([bias_scale], dtype=torch.float32, device="cuda")
    if w_pre is not None:
        w8_np, wsc = w_pre
        w_dev, w_scale_in = prequantized_device(w8_np, wsc, N, K)
        ring_w_words = ring_words(rw)
    else:
        w_dev, w_scale_in = w.cuda(), None
    if x_pre is not None:
        x8_np, xsc = x_pre
        x_dev, x_scale_in = prequantized_device(x8_np, xsc, M, K)
        ring_x_words = ring_words(rx)
    else:
        x_dev, x_scale_in = x.cuda(), None
    # outputs start as NaN: a pre-quantized operand's snapshot and zero amax
    # must be written by the library (the GEMM launch's side writes)
    scales = torch.full((4,), float("nan"), dtype=torch.float32, device="cuda")
    f = fp8.linear_forward(x_dev, w_dev, None if x_pre is not None else rx, None if w_pre is not None else rw,
                           bias=dev_bias, bias_scale=dev_bsc, x_scale_in=x_scale_in, w_scale_in=w_scale_in,
                           hist_len=rx.H, scales=scales)
    b = fp8.linear_backward(g.cuda(), f, rg, need_dbias=need_dbias)
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0

    # oracle quantize (always full) and the scale snapshots
    if x_pre is not None:
        x8o = np.zeros((M, (K + 15) // 16 * 16), np.uint8)
        x8o[:, :K] = x8_np[:, :K]
        ax, sx = np.float32(0.0), np.float32(x_pre[1])
        assert np.array_equal(ring_words(rx), ring_x_words), "ring_x must stay untouched"
    else:
        x8o, ax, sx = oracle.quantize(bits(x), oracle.DT_BF16, E4, orx, ld_out=(K + 15) // 16 * 16)
    if w_pre is not None:
        w8o, aw, sw = np.ascontiguousarray(w8_np), np.float32(0.0), np.float32(w_pre[1])
    else:
        w8o, aw, sw = oracle.quantize(bits(w), oracle.DT_BF16, E4, orw, ld_out=(K + 15) // 16 * 16)
    g8o, ag, sg = oracle.quantize(bits(g), oracle.DT_BF16, E5, org, ld_out=(N + 15) // 16 * 16)
    assert f.sx.item() == sx and f.sw.item() == sw and b.sg.item() == sg, what
    assert f.amax_x.item() == ax and f.amax_w.item() == aw and b.amax_g.item() == ag, what
    assert_codes_equal(host_rows(f.x8), x8o[:, :K], E4)
    if w_pre is None:
        assert_codes_equal(host_rows(f.w8), w8o[:, :K], E4)
    else:
        assert np.array_equal(ring_words(rw), ring_w_words), "ring_w must stay untouched"
    assert_codes_equal(host_rows(b.g8), g8o[:, :N], E5)
    if x_pre is None:
        assert np.array_equal(ring_words(rx), oracle_ring_words(orx)), what
    if w_pre is None:
        assert np.array_equal(ring_words(rw), oracle_ring_words(orw)), what
    assert np.array_equal(ring_words(rg), oracle_ring_words(org)), what
    # GEMMs (operands: the oracle's own quantized bytes, equal to the GPU's)
    gemm_check(f.y, x8o, 0, E4, w8o, E4, M, N, K, sx, sw, "fwd", full, rng, bias_np if dev_bias is not None else None,
               bias_dt, bsc, what + " y")
    gemm_check(b.dx, g8o, 0, E5, w8o, E4, M, K, N, sg, sw, "dx", full, rng, what=what + " dx")
    gemm_check(b.dw, g8o, 0, E5, x8o, E4, N, K, M, sg, sx, "dw", full, rng, what=what + " dw")
    if need_dbias:
        dbias_check(b.dbias, bits(g), M, N)
    return f, b


def make_rings(fp8, H=16):
    return (fp8.ScaleRing(H), fp8.ScaleRing(H), fp8.ScaleRing(H)), (oracle.Ring(H), oracle.Ring(H), oracle.Ring(H))


def test_config1_four_steps(fp8):
    """Config 1: 4 delayed steps, x ~ N(0,1) 2^step, w ~ N(0,0.02), bf16 bias
    ~ N(0,0.01), g ~ N(0,1e-3); full oracle comparison incl. dbias."""
    c = wl.C1
    rings, orings = make_rings(fp8)
    rng = np.random.default_rng(1)
    w = wl.normal((c.N, c.K), 0.02, wl.seed_for(1, 0, wl.OP_W))
    bias = wl.normal((c.N,), 0.01, wl.seed_for(1, 0, wl.OP_BIAS))
    for step in range(wl.C1_STEPS):
        x = wl.normal((c.M, c.K), 2.0 ** step, wl.seed_for(1, step, wl.OP_X))
        g = wl.normal((c.M, c.N), 1e-3, wl.seed_for(1, step, wl.OP_G))
        linear_step(fp8, x, w, g, rings, orings, True, rng, bias=bias, need_dbias=True, what=f"c1 step {step}")


def test_config1_no_scale_ratio_leak(fp8):
    """Two delayed steps with a doubling amax: Y at the later step stays within
    fp8 noise of the float64 GEMM of the unquantized inputs."""
    c = wl.C1
    rings, _ = make_rings(fp8)
    w = wl.normal((c.N, c.K), 0.02, wl.seed_for(1, 0, wl.OP_W))
    for step in range(3):
        x = wl.normal((c.M, c.K), 2.0 ** step, wl.seed_for(1, step, wl.OP_X))
        f = fp8.linear_forward(x.cuda(), w.cuda(), rings[0], rings[1])
        y = f.y.float().cpu().double().numpy()
        ref = x.double().numpy() @ w.double().numpy().T
        rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
        ratio = np.dot(y.ravel(), ref.ravel()) / np.dot(ref.ravel(), ref.ravel())
        assert rel < 0.25 and 0.8 < ratio < 1.2, (step, rel, ratio)


def test_prequantized_weight(fp8):
    """A pre-quantized w8 skips its quantize: amax_w = 0, sw = w_scale_in,
    ring_w untouched; config 1 shapes and config 4's path at a small size."""
    c = wl.C1
    rings, orings = make_rings(fp8)
    rng = np.random.default_rng(2)
    w = wl.normal((c.N, c.K), 0.02, wl.seed_for(1, 0, wl.OP_W))
    wsc = np.float32(448.0) / oracle.amax(bits(w), oracle.DT_BF16)
    w8 = oracle.quantize_codes(bits(w), oracle.DT_BF16, E4, wsc)
    for step in range(2):
        x = wl.normal((c.M, c.K), 1.0, wl.seed_for(1, step, wl.OP_X))
        g = wl.normal((c.M, c.N), 1e-3, wl.seed_for(1, step, wl.OP_G))
        linear_step(fp8, x, None, g, rings, orings, True, rng, w_pre=(w8, float(wsc)), what=f"w8 step {step}")


@pytest.mark.parametrize("both", (False, True), ids=("x8", "x8+w8"))
def test_prequantized_activation(fp8, both):
    """A pre-quantized x8 skips its quantize ([ops] bullet: g/x/w may each
    arrive fp8 in the matching format): sx = x_scale_in, amax_x = 0 and ring_x
    untouched, written by the GEMM launch's side writes; with w8 pre-quantized
    too no quantize runs at all and both snapshots and amaxes come from those
    side writes.  The backward then reuses the caller's x8 and scale for dW.
    Config 1 shapes (full comparison) and a c3-sized case (sampled)."""
    for (M, K, N, full, cfg) in ((wl.C1.M, wl.C1.K, wl.C1.N, True, 1), (512, 1536, 1536, False, 3)):
        rings, orings = make_rings(fp8)
        rng = np.random.default_rng(23 + cfg)
        w = wl.normal((N, K), wl.weight_std(K), wl.seed_for(cfg, 0, wl.OP_W))
        w_pre = None
        if both:
            wsc = np.float32(448.0) / oracle.amax(bits(w), oracle.DT_BF16)
            w_pre = (oracle.quantize_codes(bits(w), oracle.DT_BF16, E4, wsc), float(wsc))
        for step in range(2):
            x = wl.normal((M, K), 1.0 + step, wl.seed_for(cfg, step, wl.OP_X))
            g = wl.normal((M, N), 1e-3, wl.seed_for(cfg, step, wl.OP_G))
            xsc = np.float32(448.0) / oracle.amax(bits(x), oracle.DT_BF16) / np.float32(1.5)
            x8 = oracle.quantize_codes(bits(x), oracle.DT_BF16, E4, xsc)
            linear_step(fp8, None, None if both else w, g, rings, orings, full, rng, w_pre=w_pre,
                        x_pre=(x8, float(xsc)), need_dbias=True, what=f"x8 M={M} step {step}")


@pytest.mark.parametrize("shape", wl.C2_SHAPES, ids=lambda s: s.name)
def test_config2_shapes(fp8, shape):
    rings, orings = make_rings(fp8)
    rng = np.random.default_rng(3)
    x = wl.normal((shape.M, shape.K), 1.0, wl.seed_for(2, 0, wl.OP_X))
    w = wl.normal((shape.N, shape.K), wl.weight_std(shape.K), wl.seed_for(2, 0, wl.OP_W))
    g = wl.normal((shape.M, shape.N), 1e-3, wl.seed_for(2, 0, wl.OP_G))
    linear_step(fp8, x, w, g, rings, orings, False, rng, what=f"c2 {shape.name}")


@pytest.mark.parametrize("shape", wl.C3_SHAPES, ids=lambda s: s.name)
def test_config3_fp8_bias(fp8, shape):
    """Production shapes with the bias stored as E4M3 with bias_scale =
    448 / amax(bias), plus dbias."""
    rings, orings = make_rings(fp8)
    rng = np.random.default_rng(4)
    x = wl.normal((shape.M, shape.K), 1.0, wl.seed_for(3, 0, wl.OP_X))
    w = wl.normal((shape.N, shape.K), wl.weight_std(shape.K), wl.seed_for(3, 0, wl.OP_W))
    g = wl.normal((shape.M, shape.N), 1e-3, wl.seed_for(3, 0, wl.OP_G))
    b = wl.normal((1, shape.N), 0.01, wl.seed_for(3, 0, wl.OP_BIAS))
    bsc = np.float32(448.0) / oracle.amax(bits(b), oracle.DT_BF16)
    b8 = oracle.quantize_codes(bits(b), oracle.DT_BF16, E4, bsc)[0]
    linear_step(fp8, x, w, g, rings, orings, False, rng, bias8=b8, bias_scale=float(bsc), need_dbias=True,
                what=f"c3 {shape.name}")


@pytest.mark.parametrize("shape", wl.C4_SHAPES, ids=lambda s: s.name)
def test_config4_outliers_and_prequantized(fp8, shape):
    rings, orings = make_rings(fp8)
    rng = np.random.default_rng(5)
    x = wl.normal_with_outliers((shape.M, shape.K), 1.0, wl.seed_for(4, 0, wl.OP_X), wl.seed_for(4, 0, wl.OP_MASK))
    w = wl.normal((shape.N, shape.K), wl.weight_std(shape.K), wl.seed_for(4, 0, wl.OP_W))
    g = wl.normal((shape.M, shape.N), 1e-3, wl.seed_for(4, 0, wl.OP_G))
    linear_step(fp8, x, w, g, rings, orings, False, rng, what=f"c4 {shape.name}")
    if shape is wl.C4_SHAPES[0]:
        wsc = np.float32(448.0) / oracle.amax(bits(w), oracle.DT_BF16)
        w8 = oracle.quantize_codes(bits(w), oracle.DT_BF16, E4, wsc)
        linear_step(fp8, x, None, g, rings, orings, False, rng, w_pre=(w8, float(wsc)), what="c4 w8")


@pytest.mark.parametrize("shape", wl.C5_EDGE, ids=lambda s: s.name)
def test_config5_edge_shapes(fp8, shape):
    """Odd K (7, 100, 1534), M in {3, 64, 2048}, N in {1024, 100} (N=100 gives
    a bf16 output row of 200 bytes: the unaligned store path); bf16 bias and
    dbias; two steps."""
    rings, orings = make_rings(fp8)
    rng = np.random.default_rng(6)
    full = shape.M * shape.N * shape.K <= 64 * 1024 * 1534
    w = wl.normal((shape.N, shape.K), wl.weight_std(shape.K), wl.seed_for(5, 0, wl.OP_W))
    bias = wl.normal((shape.N,), 0.01, wl.seed_for(5, 0, wl.OP_BIAS))
    for step in range(2):
        x = wl.normal((shape.M, shape.K), 1.0 + step, wl.seed_for(5, step, wl.OP_X))
        g = wl.normal((shape.M, shape.N), 1e-3, wl.seed_for(5, step, wl.OP_G))
        linear_step(fp8, x, w, g, rings, orings, full, rng, bias=bias, need_dbias=True,
                    what=f"c5 {shape.name} step {step}")


def test_config5_twenty_step_sequence(fp8):
    """Config 5: 20 steps over 12 layers x 6 linears (216 rings), M = 2048, input
    std drifting log-uniformly in [0.5, 4] per step.  Every ring word matches
    the oracle after every step.  At every step one linear of each type (q,
    up, down) in layer step % 12 is checked in depth: x8, w8 and g8 byte for
    byte, the snapshots, and sampled y, dX and dW -- the backward dequantizing
    with the forward's snapshots."""
    H, M = wl.HIST_LEN, 2048
    words = fp8.fp8_ring_bytes(H) // 4
    nlin = wl.C5_LAYERS * len(wl.C5_LAYER)
    allbuf = torch.empty((nlin * 3, words), dtype=torch.float32, device="cuda")
    rings = [fp8.ScaleRing(H, buf=allbuf[i]) for i in range(nlin * 3)]
    orings = [oracle.Ring(H) for _ in range(nlin * 3)]
    rng = np.random.default_rng(7)
    base_x = {s.K: wl.normal((M, s.K), 1.0, wl.seed_for(5, 0, wl.OP_X, s.K)) for s in wl.C5_LAYER}
    base_g = {s.N: wl.normal((M, s.N), 1e-3, wl.seed_for(5, 0, wl.OP_G, s.N)) for s in wl.C5_LAYER}
    ws = [wl.normal((s.N, s.K), wl.weight_std(s.K), wl.seed_for(5, 0, wl.OP_W, li)) for li, s in
          enumerate(wl.C5_LAYER * wl.C5_LAYERS)]
    ws_dev = [w.cuda() for w in ws]
    w_bits = [bits(w) for w in ws]
    amax_w = [oracle.amax(b, oracle.DT_BF16) for b in w_bits]
    per_layer = len(wl.C5_LAYER)
    # one linear of each shape type within a layer: q (first), up, down
    types = [0] + [i for i, s in enumerate(wl.C5_LAYER) if s.K != s.N]
    assert len(types) == 3

    def small_sample(I, J):
        return sample_points(rng, I, J, nrows=4, ncols=4, nrand=2048)

    def check_sampled(y_dev, a8, fmt_a, a_s, b8, fmt_b, b_s, I, J, Kc, sa, sb, what):
        y = y_dev.cpu().view(torch.int16).numpy().view(np.uint16)
        pi, pj = small_sample(I, J)
        acc, sab = oracle.gemm_acc_points(pi, pj, a8, fmt_a, *a_s, b8, fmt_b, *b_s, Kc)
        want, _ = oracle.epilogue(acc, sa, sb, col_idx=pj)
        assert_gemm_close(y[pi, pj], want, sab, sa, sb, what)

    for step in range(wl.C5_STEPS):
        sigma = wl.log_uniform(0.5, 4.0, wl.seed_for(5, step, wl.OP_STD))
        xs = {K: (t.float() * sigma).to(torch.bfloat16) for K, t in base_x.items()}
        gs = {N: (t.float() * (sigma / 2)).to(torch.bfloat16) for N, t in base_g.items()}
        xs_dev = {K: t.cuda() for K, t in xs.items()}
        gs_dev = {N: t.cuda() for N, t in gs.items()}
        xa = {K: oracle.amax(bits(t), oracle.DT_BF16) for K, t in xs.items()}
        ga = {N: oracle.amax(bits(t), oracle.DT_BF16) for N, t in gs.items()}
        deep = {(step % wl.C5_LAYERS) * per_layer + t for t in types}
        for li, s in enumerate(wl.C5_LAYER * wl.C5_LAYERS):
            rx, rw, rg = rings[3 * li: 3 * li + 3]
            f = fp8.linear_forward(xs_dev[s.K], ws_dev[li], rx, rw)
            b = fp8.linear_backward(gs_dev[s.N], f, rg)
            orx, orw, org = orings[3 * li: 3 * li + 3]
            sx, sw, sg = orx.scale, orw.scale, org.scale
            orx.advance(xa[s.K], E4)
            orw.advance(amax_w[li], E4)
            org.advance(ga[s.N], E5)
            if li in deep:
                torch.cuda.synchronize()
                what = f"c5 step {step} linear {li} ({s.name})"
                assert (f.sx.item(), f.sw.item(), b.sg.item()) == (sx, sw, sg), what
                assert (f.amax_x.item(), f.amax_w.item(), b.amax_g.item()) == (xa[s.K], amax_w[li], ga[s.N]), what
                x8 = oracle.quantize_codes(bits(xs[s.K]), oracle.DT_BF16, E4, sx)
                w8 = oracle.quantize_codes(w_bits[li], oracle.DT_BF16, E4, sw)
                g8 = oracle.quantize_codes(bits(gs[s.N]), oracle.DT_BF16, E5, sg)
                assert_codes_equal(host_rows(f.x8), x8, E4)
                assert_codes_equal(host_rows(f.w8), w8, E4)
                assert_codes_equal(host_rows(b.g8), g8, E5)
                K, N = s.K, s.N
                check_sampled(f.y, x8, E4, (K, 1), w8, E4, (K, 1), M, N, K, sx, sw, what + " y")
                check_sampled(b.dx, g8, E5, (N, 1), w8, E4, (1, K), M, K, N, sg, sw, what + " dx")
                check_sampled(b.dw, g8, E5, (1, N), x8, E4, (1, K), N, K, M, sg, sx, what + " dw")
        torch.cuda.synchronize()
        got = allbuf.cpu().view(torch.int32).numpy().view(np.uint32)
        want = np.stack([oracle_ring_words(r) for r in orings])
        assert np.array_equal(got, want), f"ring words differ at step {step}"
    assert fp8.fp8_get_device_status() == 0


@pytest.mark.parametrize("dtype", (torch.float16, torch.float32))
@pytest.mark.parametrize("M,N,K", [(300, 100, 64), (1000, 1000, 128), (2048, 1536, 256)])
def test_backward_fused_colsum_dtypes(fp8, dtype, M, N, K):
    """g in fp16/fp32 (odd N, ragged row splits): the quantize-with-column-sum
    launch gives bit-exact g8/ring and dbias within max(1 ulp, 2e-6 sum|g|)."""
    rng = np.random.default_rng(M + N)
    rx, rw, rg = fp8.ScaleRing(16), fp8.ScaleRing(16), fp8.ScaleRing(16)
    org = oracle.Ring(16)
    x = wl.normal((M, K), 1.0, 11, dtype=torch.bfloat16)
    w = wl.normal((N, K), 0.05, 12, dtype=torch.bfloat16)
    f = fp8.linear_forward(x.cuda(), w.cuda(), rx, rw)
    for step in range(2):
        g = wl.normal((M, N), 1e-3 * (1 + step), 13 + step, dtype=dtype)
        b = fp8.linear_backward(g.cuda(), f, rg, need_dx=False, need_dw=False, need_dbias=True)
        torch.cuda.synchronize()
        gb = bits(g)
        dt = oracle.DT_FP16 if dtype == torch.float16 else oracle.DT_FP32
        g8o, ag, sg = oracle.quantize(gb, dt, E5, org, ld_out=(N + 15) // 16 * 16)
        assert b.sg.item() == sg and b.amax_g.item() == ag
        assert_codes_equal(host_rows(b.g8), g8o[:, :N], E5)
        assert np.array_equal(ring_words(rg), oracle_ring_words(org))
        want, _, sa = oracle.dbias(gb, dt, M, N)
        gv = oracle.bf16_to_f32(b.dbias.cpu().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
        ov = oracle.bf16_to_f32(want).astype(np.float64)
        assert np.all(np.abs(gv - ov) <= np.maximum(oracle.bf16_ulp(ov), 2e-6 * sa))
    assert fp8.fp8_get_device_status() == 0


@pytest.mark.parametrize("need_dx,need_dw", [(True, False), (False, True)])
@pytest.mark.parametrize("need_dbias", [False, True])
def test_backward_need_masks(fp8, need_dx, need_dw, need_dbias):
    """dX alone or dW alone: the backward's one GEMM launch (instead of the
    dX + dW pair) also completes the g ring's step and, with the bias
    gradient, the column sums.  Over two steps g8, the snapshot, amax and
    every ring word are bit-exact, the requested gradient is within the GEMM
    tolerance in full, and the buffer of the gradient not requested is left
    as it was."""
    rng = np.random.default_rng(7 + int(need_dx) + 2 * int(need_dbias))
    M, N, K = 700, 520, 384
    rx, rw, rg = fp8.ScaleRing(16), fp8.ScaleRing(16), fp8.ScaleRing(16)
    org = oracle.Ring(16)
    x = wl.normal((M, K), 1.0, 41)
    w = wl.normal((N, K), 0.05, 42)
    f = fp8.linear_forward(x.cuda(), w.cuda(), rx, rw)
    torch.cuda.synchronize()
    x8, w8 = host_rows(f.x8), host_rows(f.w8)
    dx = torch.full((M, K), 7.0, dtype=torch.bfloat16, device="cuda")
    dw = torch.full((N, K), 7.0, dtype=torch.bfloat16, device="cuda")
    for step in range(2):
        g = wl.normal((M, N), 1e-3 * (1 + 2 * step), 43 + step)
        b = fp8.linear_backward(g.cuda(), f, rg, need_dx=need_dx, need_dw=need_dw, need_dbias=need_dbias,
                                dx=dx, dw=dw)
        torch.cuda.synchronize()
        gb = bits(g)
        g8o, ag, sg = oracle.quantize(gb, oracle.DT_BF16, E5, org, ld_out=(N + 15) // 16 * 16)
        assert b.sg.item() == sg and b.amax_g.item() == ag
        g8c = np.ascontiguousarray(g8o[:, :N])
        assert_codes_equal(host_rows(b.g8), g8c, E5)
        assert np.array_equal(ring_words(rg), oracle_ring_words(org))
        what = f"step {step} need_dx={need_dx} need_dw={need_dw} need_dbias={need_dbias}"
        if need_dx:
            gemm_check(dx, g8c, 0, E5, w8, E4, M, K, N, sg, f.sw.item(), "dx", True, rng, what=what + " dx")
        else:
            assert bool((dx == 7.0).all()), what
        if need_dw:
            gemm_check(dw, g8c, 0, E5, x8, E4, N, K, M, sg, f.sx.item(), "dw", True, rng, what=what + " dw")
        else:
            assert bool((dw == 7.0).all()), what
        if need_dbias:
            dbias_check(b.dbias, gb, M, N)
    assert fp8.fp8_get_device_status() == 0


def test_backward_prequantized_g_dbias(fp8):
    """A pre-quantized g (E5M2 codes with its scale) skips its quantize
    (sg = g_scale_in, amax_g = 0, ring untouched) and dbias dequantizes each
    element before the sum."""
    rng = np.random.default_rng(21)
    M, N, K = 512, 384, 256
    rx, rw, rg = fp8.ScaleRing(16), fp8.ScaleRing(16), fp8.ScaleRing(16)
    x = wl.normal((M, K), 1.0, 31)
    w = wl.normal((N, K), 0.05, 32)
    f = fp8.linear_forward(x.cuda(), w.cuda(), rx, rw)
    g = wl.normal((M, N), 1e-3, 33)
    sg = np.float32(57344.0) / oracle.amax(bits(g), oracle.DT_BF16)
    g8 = oracle.quantize_codes(bits(g), oracle.DT_BF16, E5, sg)
    before = ring_words(rg)
    gdev = torch.from_numpy(g8).cuda()
    sgd = torch.tensor([float(sg)], device="cuda")
    b = fp8.linear_backward(gdev, f, rg, need_dbias=True, g_scale_in=sgd)
    torch.cuda.synchronize()
    assert b.sg.item() == sg and b.amax_g.item() == 0.0
    assert np.array_equal(ring_words(rg), before)
    want, _, sa = oracle.dbias(g8, oracle.DT_E5M2, M, N, sg)
    gv = oracle.bf16_to_f32(b.dbias.cpu().view(torch.int16).numpy().view(np.uint16)).astype(np.float64)
    ov = oracle.bf16_to_f32(want).astype(np.float64)
    assert np.all(np.abs(gv - ov) <= np.maximum(oracle.bf16_ulp(ov), 2e-6 * sa))
    torch.cuda.synchronize()
    x8 = host_rows(f.x8)
    w8 = host_rows(f.w8)
    gemm_check(b.dx, g8, 0, E5, w8, E4, M, K, N, sg, f.sw.item(), "dx", True, rng, what="pre-g dx")
    gemm_check(b.dw, g8, 0, E5, x8, E4, N, K, M, sg, f.sx.item(), "dw", True, rng, what="pre-g dw")


def test_forward_mixed_input_dtypes(fp8):
    """x fp32 and w bf16 (no shared launch): two quantize launches, same results
    as the oracle."""
    rng = np.random.default_rng(22)
    M, N, K = 256, 320, 192
    rx, rw = fp8.ScaleRing(16), fp8.ScaleRing(16)
    orx, orw = oracle.Ring(16), oracle.Ring(16)
    for step in range(2):
        x = wl.normal((M, K), 1.0 + step, 41 + step, dtype=torch.float32)
        w = wl.normal((N, K), 0.05, 43)
        f = fp8.linear_forward(x.cuda(), w.cuda(), rx, rw)
        torch.cuda.synchronize()
        x8o, ax, sx = oracle.quantize(bits(x), oracle.DT_FP32, E4, orx)
        w8o, aw, sw = oracle.quantize(bits(w), oracle.DT_BF16, E4, orw)
        assert (f.sx.item(), f.sw.item(), f.amax_x.item(), f.amax_w.item()) == (sx, sw, ax, aw)
        assert_codes_equal(host_rows(f.x8), x8o, E4)
        assert np.array_equal(ring_words(rx), oracle_ring_words(orx))
        gemm_check(f.y, x8o, 0, E4, w8o, E4, M, N, K, sx, sw, "fwd", True, rng, what="mixed y")


@pytest.mark.parametrize("M,N,K", [(64, 192, 0), (0, 192, 128), (64, 0, 128), (0, 0, 0)],
                         ids=["K0", "M0", "N0", "all0"])
@pytest.mark.parametrize("bias_kind", ("bf16", "e4m3"))
def test_empty_sizes(fp8, M, N, K, bias_kind):
    """Empty sizes: an operand with no elements is not quantized (its ring does
    not step); a non-empty one is, with its ring step; y is the bias when the
    contraction K is empty; a requested gradient with elements is zero when its
    contraction is empty (dX when N = 0, dW and dbias when M = 0) and dbias is
    the column sum of g when K = 0 -- all against the oracle's orchestration."""
    rx, rw, rg = fp8.ScaleRing(16), fp8.ScaleRing(16), fp8.ScaleRing(16)
    orx, orw, org = oracle.Ring(16), oracle.Ring(16), oracle.Ring(16)
    x = wl.normal((M, K), 1.0, 61)
    w = wl.normal((N, K), 0.05, 62)
    g = wl.normal((M, N), 1e-3, 63)
    b = wl.normal((N,), 0.01, 64)
    if bias_kind == "bf16":
        dev_bias, dev_bsc, bias_np, bias_dt, bsc = b.cuda(), None, bits(b), oracle.DT_BF16, 1.0
    else:
        bsc = np.float32(448.0) / max(oracle.amax(bits(b).reshape(1, -1), oracle.DT_BF16), np.float32(1e-3)) \
            if N else np.float32(1.0)
        b8 = oracle.quantize_codes(bits(b).reshape(1, -1), oracle.DT_BF16, E4, bsc)[0] if N else \
            np.zeros(0, np.uint8)
        dev_bias, dev_bsc = torch.from_numpy(np.ascontiguousarray(b8)).cuda(), \
            torch.tensor([float(bsc)], device="cuda")
        bias_np, bias_dt = b8, oracle.DT_E4M3
    before = [ring_words(r).copy() for r in (rx, rw, rg)]
    f = fp8.linear_forward(x.cuda(), w.cuda(), rx, rw, bias=dev_bias, bias_scale=dev_bsc)
    bwd = fp8.linear_backward(g.cuda(), f, rg, need_dbias=True)
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0
    of = oracle.linear_forward(M, N, K, bits(x), oracle.DT_BF16, bits(w), oracle.DT_BF16, orx, orw,
                               bias=bias_np, bias_dtype=bias_dt, bias_scale=float(bsc),
                               ldx8=(K + 15) // 16 * 16, ldw8=(K + 15) // 16 * 16)
    ob = oracle.linear_backward(M, N, K, bits(g), oracle.DT_BF16, org, of["x8"], E4, of["sx"], of["w8"], E4,
                                of["sw"], ldg8=(N + 15) // 16 * 16, need_dbias=True)
    # rings: stepped exactly when their operand has elements
    for ring, oring, live, b0 in ((rx, orx, M * K > 0, before[0]), (rw, orw, N * K > 0, before[1]),
                                  (rg, org, M * N > 0, before[2])):
        if live:
            assert np.array_equal(ring_words(ring), oracle_ring_words(oring))
        else:
            assert np.array_equal(ring_words(ring), b0) and oring.step == 0
    if M * K:
        assert_codes_equal(host_rows(f.x8), of["x8"][:, :K], E4)
        assert f.sx.item() == of["sx"] and f.amax_x.item() == of["amax_x"]
    if N * K:
        assert_codes_equal(host_rows(f.w8), of["w8"][:, :K], E4)
        assert f.sw.item() == of["sw"] and f.amax_w.item() == of["amax_w"]
    if M * N:
        assert_codes_equal(host_rows(bwd.g8), ob["g8"][:, :N], E5)
        y = f.y.cpu().view(torch.int16).numpy().view(np.uint16)
        assert_gemm_close(y, of["y"], np.zeros(of["y"].shape), 1.0, 1.0, "y of an empty contraction")
    if M * K:
        assert np.array_equal(bwd.dx.cpu().view(torch.int16).numpy().view(np.uint16), ob["dx"])
    if N * K:
        assert np.array_equal(bwd.dw.cpu().view(torch.int16).numpy().view(np.uint16), ob["dw"])
    if N:
        got = bwd.dbias.cpu().view(torch.int16).numpy().view(np.uint16)
        gv, ov = oracle.bf16_to_f32(got).astype(np.float64), oracle.bf16_to_f32(ob["dbias"]).astype(np.float64)
        assert np.all(np.abs(gv - ov) <= np.maximum(oracle.bf16_ulp(ov), 2e-6 * ob["dbias_sumabs"]))


def test_nan_inputs_propagate(fp8):
    """NaN elements in x and g: amax ignores them (rings step on the finite
    values), they cast to the NaN code, and the NaN reaches exactly the GEMM
    outputs and bias-gradient columns whose sums contain it -- row r of y, row
    r of dX and row j of dW (g's NaN at (r, j)), column c of dW (x's NaN at
    column c), entry j of dbias -- as in
    the oracle."""
    rng = np.random.default_rng(41)
    M, K, N = 384, 320, 272
    x = wl.normal((M, K), 1.0, 4101)
    w = wl.normal((N, K), 0.05, 4102)
    g = wl.normal((M, N), 1e-3, 4103)
    x[17, 5] = float("nan")
    x[300, 250] = float("nan")
    g[40, 7] = float("nan")
    bias = wl.normal((N,), 0.01, 4104)
    rings, orings = make_rings(fp8)
    f, b = linear_step(fp8, x, w, g, rings, orings, True, rng, bias=bias, need_dbias=True, what="nan inputs")
    y = f.y.float().cpu()
    dx, dw, db = b.dx.float().cpu(), b.dw.float().cpu(), b.dbias.float().cpu()
    assert torch.isnan(y[17]).all() and torch.isnan(y[300]).all() and not torch.isnan(y[18]).any()
    assert torch.isnan(dw[:, 5]).all() and torch.isnan(dw[:, 250]).all() and torch.isnan(dw[7]).all()
    assert torch.isnan(dx[40]).all() and not torch.isnan(dx[41]).any()
    assert torch.isnan(db[7]) and not torch.isnan(db[8])
