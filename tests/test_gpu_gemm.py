"""GPU parity of the FP8 GEMM primitive (fp8_mm) against the oracle, for all
four operand layouts (the forward's K-major x K-major, dX's K-major x MN-major,
dW's MN-major x MN-major, and MN-major x K-major), ragged and multi-tile
shapes, both fp8 formats and the bias variants.  Tolerance per element:
max(1 bf16 ulp of the oracle value, 2e-6 sum_k |a_k b_k| / (sa sb))."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_gemm_close, sample_points

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def codes_like_tensor(rng, fmt, shape, std):
    """fp8 codes of a normal tensor scaled into the format's range (oracle cast)."""
    v = (rng.standard_normal(shape) * std).astype(np.float32)
    return oracle.encode(fmt, v)


def store(codes_logical, major, pad):
    """Logical [I, Kc] operand -> storage array with row stride ld: K-major
    [I, ld >= Kc], MN-major [Kc, ld >= I].  Padding bytes hold junk (0x77)."""
    mat = codes_logical if major == 0 else np.ascontiguousarray(codes_logical.T)
    rows, cols = mat.shape
    ld = (cols + 15) // 16 * 16 + pad
    buf = np.full((rows, ld), 0x77, np.uint8)
    buf[:, :cols] = mat
    return buf, ld


def strides(major, ld):
    return (ld, 1) if major == 0 else (1, ld)


def run_case(fp8, rng, m, n, k, a_major, b_major, fmt_a=0, fmt_b=0, sa=1.0, sb=1.0, bias_kind=None,
             pad=0, ldd_extra=0, full=True, a_codes=None, b_codes=None, tile=0, workspace=None):
    A = a_codes if a_codes is not None else codes_like_tensor(rng, fmt_a, (m, k), 60.0 if fmt_a == 0 else 3000.0)
    B = b_codes if b_codes is not None else codes_like_tensor(rng, fmt_b, (n, k), 60.0 if fmt_b == 0 else 3000.0)
    a_st, lda = store(A, a_major, pad)
    b_st, ldb = store(B, b_major, pad)
    dev_a = torch.from_numpy(a_st).cuda()
    dev_b = torch.from_numpy(b_st).cuda()
    scales = torch.tensor([sa, sb], dtype=torch.float32, device="cuda")
    ldd = n + ldd_extra
    d = torch.full((m, ldd), float("nan"), dtype=torch.bfloat16, device="cuda")
    bias = bias_dev = bias_scale = None
    bias_dtype = fp8.FP8_DT_BF16
    bsc = 1.0
    if bias_kind == "bf16":
        bias = torch.from_numpy((rng.standard_normal(n) * 5).astype(np.float32)).to(torch.bfloat16)
        bias_dev = bias.cuda()
        bias_np = bias.view(torch.int16).numpy().view(np.uint16)
        odt = oracle.DT_BF16
    elif bias_kind in ("e4m3", "e5m2"):
        bf = 0 if bias_kind == "e4m3" else 1
        bias_np = codes_like_tensor(rng, bf, (n,), 100.0)
        bias_dev = torch.from_numpy(bias_np).cuda()
        bsc = 7.25
        bias_scale = torch.tensor([bsc], dtype=torch.float32, device="cuda")
        bias_dtype = fp8.FP8_DT_E4M3 + bf
        odt = oracle.DT_E4M3 + bf
    fp8.fp8_mm(m, n, k, dev_a, fmt_a, a_major, lda, dev_b, fmt_b, b_major, ldb, scales[0:1], scales[1:2], d, ldd,
               bias=bias_dev, bias_dtype=bias_dtype, bias_scale=bias_scale, tile_cfg=tile, workspace=workspace)
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0
    y = d.cpu().view(torch.int16).numpy().view(np.uint16)
    if ldd_extra:
        assert np.all(y[:, n:] == 0x7FC0), "bytes past n must stay untouched"
        y = y[:, :n]
    a_si, a_sk = strides(a_major, lda)
    b_sj, b_sk = strides(b_major, ldb)
    if full:
        acc, _, sab = oracle.gemm_acc(a_st, fmt_a, a_si, a_sk, b_st, fmt_b, b_sj, b_sk, m, n, k)
        want, _ = oracle.epilogue(acc, sa, sb, bias_np if bias_kind else None,
                                  odt if bias_kind else 0, bsc)
        return assert_gemm_close(y, want, sab, sa, sb, f"mm {m}x{n}x{k} {a_major}{b_major}"), y, want
    pi, pj = sample_points(rng, m, n)
    acc, sab = oracle.gemm_acc_points(pi, pj, a_st, fmt_a, a_si, a_sk, b_st, fmt_b, b_sj, b_sk, k)
    want, _ = oracle.epilogue(acc, sa, sb, bias_np if bias_kind else None, odt if bias_kind else 0, bsc,
                              col_idx=pj)
    return assert_gemm_close(y[pi, pj], want, sab, sa, sb, f"mm {m}x{n}x{k} {a_major}{b_major} sampled"), y, None


LAYOUTS = [(0, 0), (0, 1), (1, 1), (1, 0)]
# 128x128, 128x256 (one CTA), 256x256 (CTA pair, 2-SM MMA), 128x128 split-K
# over a cluster (forced: S = 2..3 by k-blocks and residency; one k-block runs unsplit)
TILES = [1, 2, 3, 4]


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("a_major,b_major", LAYOUTS)
@pytest.mark.parametrize("m,n,k", [(64, 192, 128), (128, 256, 256), (200, 300, 333), (3, 100, 7),
                                   (1000, 700, 1040), (130, 129, 2000), (600, 520, 384)])
def test_mm_layouts_full(fp8, a_major, b_major, m, n, k, tile):
    rng = np.random.default_rng(m * 7 + n * 3 + k + 10 * a_major + b_major)
    run_case(fp8, rng, m, n, k, a_major, b_major, sa=448.0 / 300, sb=0.75, pad=16 if m == 200 else 0, tile=tile)


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("fmt_a,fmt_b", [(1, 0), (1, 1), (0, 1)])
@pytest.mark.parametrize("a_major,b_major", LAYOUTS)
def test_mm_formats(fp8, fmt_a, fmt_b, a_major, b_major, tile):
    rng = np.random.default_rng(99 + fmt_a * 2 + fmt_b)
    run_case(fp8, rng, 257, 384, 640, a_major, b_major, fmt_a, fmt_b, sa=57344.0 / 9000, sb=448.0 / 200, tile=tile)


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("bias_kind", ["bf16", "e4m3", "e5m2"])
def test_mm_bias(fp8, bias_kind, tile):
    rng = np.random.default_rng(5)
    run_case(fp8, rng, 300, 500, 384, 0, 0, sa=2.0, sb=3.0, bias_kind=bias_kind, tile=tile)
    run_case(fp8, rng, 64, 100, 96, 0, 0, sa=1.0, sb=1.0, bias_kind=bias_kind, ldd_extra=4, tile=tile)


@pytest.mark.parametrize("tile", TILES)
def test_mm_odd_ldd_untouched_columns(fp8, tile):
    rng = np.random.default_rng(6)
    run_case(fp8, rng, 129, 100, 128, 0, 1, ldd_extra=3, tile=tile)
    run_case(fp8, rng, 77, 264, 300, 1, 1, ldd_extra=8, tile=tile)
    run_case(fp8, rng, 300, 264, 300, 0, 0, ldd_extra=8, tile=tile)


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("a_major,b_major", LAYOUTS)
def test_mm_small_integers_exact(fp8, a_major, b_major, tile):
    """Small-integer fp8 values with unit scales: every partial sum is an integer
    below 2^24, so the GPU must equal the oracle (and the integer matmul) bit
    for bit."""
    rng = np.random.default_rng(7)
    t = oracle.decode_table(0)
    ints = np.array([c for c in range(256) if np.isfinite(t[c]) and t[c] == np.round(t[c]) and abs(t[c]) <= 4],
                    np.uint8)
    m, n, k = 300, 520, 1000
    A = rng.choice(ints, size=(m, k))
    B = rng.choice(ints, size=(n, k))
    _, y, want = run_case(fp8, rng, m, n, k, a_major, b_major, a_codes=A, b_codes=B, tile=tile)
    ref = (t[A].astype(np.int64) @ t[B].astype(np.int64).T).astype(np.float32)
    assert np.array_equal(oracle.bf16_to_f32(y), oracle.bf16_to_f32(want))
    assert np.array_equal(oracle.bf16_to_f32(y), oracle.bf16_to_f32(oracle.bf16_rne(ref)))


def test_mm_identity_weight(fp8):
    """W8 = identity: Y = bf16(decode(x8) / (sx sw)) (bf16 rounding of one product)."""
    rng = np.random.default_rng(8)
    K = 384
    A = codes_like_tensor(rng, 0, (256, K), 100.0)
    B = np.where(np.eye(K, dtype=bool), 0x38, 0x00).astype(np.uint8)
    run_case(fp8, rng, 256, K, K, 0, 0, a_codes=A, b_codes=B, sa=0.5, sb=1.0)
    run_case(fp8, rng, 256, K, K, 0, 1, a_codes=A, b_codes=B, sa=0.5, sb=1.0)


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("a_major,b_major", LAYOUTS)
def test_mm_long_k_accumulation(fp8, a_major, b_major, tile):
    """K = 11008 (the longest contraction of the workloads): random signs and
    all-positive operands.  The all-positive case bounds the accumulation error
    of the tensor-core path against the exact dot."""
    rng = np.random.default_rng(9)
    run_case(fp8, rng, 256, 256, 11008, a_major, b_major, sa=448.0 / 200, sb=448.0 / 150, tile=tile)
    pos = oracle.encode(0, np.abs(rng.standard_normal((128, 11008)) * 30).astype(np.float32) + 1.0)
    posb = oracle.encode(0, np.abs(rng.standard_normal((256, 11008)) * 30).astype(np.float32) + 1.0)
    run_case(fp8, rng, 128, 256, 11008, a_major, b_major, a_codes=pos, b_codes=posb, tile=tile)


@pytest.mark.parametrize("tile", [0] + TILES)
@pytest.mark.parametrize("m,n,k,a_major,b_major", [
    (2048, 1024, 1024, 0, 0), (2048, 1024, 4096, 0, 1), (4096, 1024, 2048, 1, 1), (512, 6912, 1536, 0, 0),
    (1536, 1536, 512, 1, 1), (640, 2304, 4096, 0, 0), (4096, 11008, 512, 0, 0),
    (512, 1536, 6912, 0, 0), (512, 1536, 6912, 0, 1), (512, 1536, 1536, 1, 1)])
def test_mm_large_sampled(fp8, m, n, k, a_major, b_major, tile):
    rng = np.random.default_rng(m + n + k)
    run_case(fp8, rng, m, n, k, a_major, b_major, sa=3.0, sb=0.25, full=False, tile=tile)


def test_mm_no_device_timeouts(fp8):
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0


@pytest.mark.parametrize("tile", [0] + TILES)
def test_mm_pair_matches_two_calls(fp8, tile):
    """fp8_mm_pair runs dX-like (K x MN-major) and dW-like (MN x MN-major) GEMMs
    of different shapes in one launch; each output equals its own fp8_mm call
    with the same tile configuration bit for bit (split-K, which two-GEMM
    launches do not use, against the 128x128 fallback)."""
    rng = np.random.default_rng(31)
    M, N, K = 700, 520, 300
    g8 = codes_like_tensor(rng, 1, (M, N), 3000.0)
    w8 = codes_like_tensor(rng, 0, (N, K), 60.0)
    x8 = codes_like_tensor(rng, 0, (M, K), 60.0)
    gs, ldg = store(g8, 0, 0)
    ws, ldw = store(w8, 0, 0)
    xs, ldx = store(x8, 0, 0)
    G, W, X = (torch.from_numpy(t).cuda() for t in (gs, ws, xs))
    sc = torch.tensor([3.0, 0.5, 0.25], device="cuda")
    dx1 = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dw1 = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    dx2, dw2 = torch.empty_like(dx1), torch.empty_like(dw1)
    p = lambda t: t.data_ptr()  # noqa: E731
    s4 = sc.data_ptr()

    def args(dx, dw, cfg):
        a = fp8.MmArgs(M, K, N, p(G), 1, 0, ldg, p(W), 0, 1, ldw, s4, s4 + 4, None, 0, None, p(dx), K, cfg)
        b = fp8.MmArgs(N, K, M, p(G), 1, 1, ldg, p(X), 0, 1, ldx, s4, s4 + 8, None, 0, None, p(dw), K, cfg)
        return a, b
    a, b = args(dx1, dw1, tile)
    fp8.fp8_mm_pair(a, b)
    torch.cuda.synchronize()
    if tile == 0:
        # auto picks one config for the pair; check against the oracle instead
        gemm_dx, _, sab = oracle.gemm_acc(gs, 1, ldg, 1, ws, 0, 1, ldw, M, K, N)
        want, _ = oracle.epilogue(gemm_dx, 3.0, 0.5)
        assert_gemm_close(dx1.cpu().view(torch.int16).numpy().view(np.uint16), want, sab, 3.0, 0.5, "pair dx")
        gemm_dw, _, sab = oracle.gemm_acc(gs, 1, 1, ldg, xs, 0, 1, ldx, N, K, M)
        want, _ = oracle.epilogue(gemm_dw, 3.0, 0.25)
        assert_gemm_close(dw1.cpu().view(torch.int16).numpy().view(np.uint16), want, sab, 3.0, 0.25, "pair dw")
    else:
        # a two-GEMM launch does not split K: forced split-K falls back to 128x128
        a2, b2 = args(dx2, dw2, 1 if tile == 4 else tile)
        fp8._lib.fp8_mm(ctypes.byref(a2), torch.cuda.current_stream().cuda_stream)
        fp8._lib.fp8_mm(ctypes.byref(b2), torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        assert torch.equal(dx1.view(torch.int16), dx2.view(torch.int16))
        assert torch.equal(dw1.view(torch.int16), dw2.view(torch.int16))
    assert fp8.fp8_get_device_status() == 0


@pytest.mark.parametrize("m,n,k,a_major,b_major", [(300, 260, 1000, 0, 0), (512, 1536, 6912, 0, 1)])
def test_mm_split_k_deterministic(fp8, m, n, k, a_major, b_major):
    """Split-K sums the ranks' partials in rank order, so two launches give the
    same bits; and AUTO on a few-tile, long-K shape agrees with forced split-K
    within the GEMM tolerance (AUTO may or may not split)."""
    rng = np.random.default_rng(77)
    _, y1, _ = run_case(fp8, rng, m, n, k, a_major, b_major, full=False, tile=4)
    rng = np.random.default_rng(77)
    _, y2, _ = run_case(fp8, rng, m, n, k, a_major, b_major, full=False, tile=4)
    assert np.array_equal(y1, y2)


# ---------------------------------------------------------------- batched (3-D) GEMMs

def stack_operand(mats, major):
    """Per-batch logical operands -> one storage array of the batches one after
    another, its row stride and its batch stride (elements)."""
    sts = [store(x, major, 0) for x in mats]
    rows, ld = sts[0][0].shape
    return np.concatenate([s_ for s_, _ in sts], axis=0), ld, rows * ld, [s_ for s_, _ in sts]


def run_batched(fp8, rng, batch, m, n, k, a_major, b_major, bcast_a=False, bcast_b=False, tile=0, bias=False,
                d_gap=0, full=True):
    As = [codes_like_tensor(rng, 0, (m, k), 60.0) for _ in range(1 if bcast_a else batch)]
    Bs = [codes_like_tensor(rng, 1, (n, k), 3000.0) for _ in range(1 if bcast_b else batch)]
    a_buf, lda, sa, a_sts = stack_operand(As, a_major)
    b_buf, ldb, sb, b_sts = stack_operand(Bs, b_major)
    ldd = n + (8 if d_gap else 0)
    sd = m * ldd + d_gap
    dflat = torch.full((batch * sd,), float("nan"), dtype=torch.bfloat16, device="cuda")
    A, B = torch.from_numpy(a_buf).cuda(), torch.from_numpy(b_buf).cuda()
    sc = torch.tensor([2.5, 0.125], dtype=torch.float32, device="cuda")
    bias_np = bias_dev = None
    if bias:
        bt = torch.from_numpy((rng.standard_normal(n) * 3).astype(np.float32)).to(torch.bfloat16)
        bias_dev, bias_np = bt.cuda(), bt.view(torch.int16).numpy().view(np.uint16)
    args = fp8.MmArgs(m, n, k, A.data_ptr(), 0, a_major, lda, B.data_ptr(), 1, b_major, ldb, sc.data_ptr(),
                      sc.data_ptr() + 4, bias_dev.data_ptr() if bias else None, 0, None, dflat.data_ptr(), ldd, tile)
    fp8.fp8_mm_batched(args, batch, 0 if bcast_a else sa, 0 if bcast_b else sb, sd)
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0
    allbits = dflat.cpu().view(torch.int16).numpy().view(np.uint16)
    a_si, a_sk = strides(a_major, lda)
    b_sj, b_sk = strides(b_major, ldb)
    outs = []
    for bi in range(batch):
        blk = allbits[bi * sd: bi * sd + m * ldd].reshape(m, ldd)
        y = blk[:, :n]
        if ldd > n:
            assert np.all(blk[:, n:] == 0x7FC0), "columns past n must stay untouched"
        if d_gap:
            assert np.all(allbits[bi * sd + m * ldd: (bi + 1) * sd] == 0x7FC0), "gap between batches untouched"
        a_st = a_sts[0 if bcast_a else bi]
        b_st = b_sts[0 if bcast_b else bi]
        if full:
            acc, _, sab = oracle.gemm_acc(a_st, 0, a_si, a_sk, b_st, 1, b_sj, b_sk, m, n, k)
            want, _ = oracle.epilogue(acc, 2.5, 0.125, bias_np, oracle.DT_BF16 if bias else 0)
            assert_gemm_close(y, want, sab, 2.5, 0.125, f"batched b={bi}")
        else:
            pi, pj = sample_points(rng, m, n)
            acc, sab = oracle.gemm_acc_points(pi, pj, a_st, 0, a_si, a_sk, b_st, 1, b_sj, b_sk, k)
            want, _ = oracle.epilogue(acc, 2.5, 0.125, bias_np, oracle.DT_BF16 if bias else 0, col_idx=pj)
            assert_gemm_close(y[pi, pj], want, sab, 2.5, 0.125, f"batched b={bi} sampled")
        outs.append(y.copy())
    return outs


@pytest.mark.parametrize("tile", [0, 1, 2, 3])
@pytest.mark.parametrize("a_major,b_major", LAYOUTS)
def test_mm_batched_layouts(fp8, a_major, b_major, tile):
    """Three batches of a ragged shape, every layout and tile configuration,
    a padded output row stride and a gap between the batches' outputs."""
    rng = np.random.default_rng(50 + 4 * a_major + b_major + 10 * tile)
    run_batched(fp8, rng, 3, 200, 300, 333, a_major, b_major, tile=tile, bias=True, d_gap=24)


@pytest.mark.parametrize("bcast_a,bcast_b", [(False, True), (True, False)])
@pytest.mark.parametrize("a_major,b_major", [(0, 0), (0, 1), (1, 1)])
def test_mm_batched_broadcast(fp8, a_major, b_major, bcast_a, bcast_b):
    """A zero batch stride shares that operand across the batch (the pages'
    size-1 batch broadcast): a shared weight, or a shared activation."""
    rng = np.random.default_rng(60 + a_major + 2 * b_major + 4 * bcast_a)
    run_batched(fp8, rng, 4, 130, 257, 200, a_major, b_major, bcast_a=bcast_a, bcast_b=bcast_b)


def test_mm_batched_single_equals_mm(fp8):
    """batch = 1 is fp8_mm bit for bit; a batch whose matrices are copies of one
    operand pair gives identical outputs."""
    rng = np.random.default_rng(70)
    m, n, k = 300, 260, 1000
    A8 = codes_like_tensor(rng, 0, (m, k), 60.0)
    B8 = codes_like_tensor(rng, 1, (n, k), 3000.0)
    a_st, lda = store(A8, 0, 0)
    b_st, ldb = store(B8, 0, 0)
    A, B = torch.from_numpy(a_st).cuda(), torch.from_numpy(b_st).cuda()
    A3 = torch.from_numpy(np.concatenate([a_st] * 3)).cuda()
    sc = torch.tensor([1.5, 0.5], dtype=torch.float32, device="cuda")
    d1 = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    d2 = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    d3 = torch.empty((3, m, n), dtype=torch.bfloat16, device="cuda")
    mk = lambda a_, d_: fp8.MmArgs(m, n, k, a_.data_ptr(), 0, 0, lda, B.data_ptr(), 1, 0, ldb,  # noqa: E731
                                   sc.data_ptr(), sc.data_ptr() + 4, None, 0, None, d_.data_ptr(), n, 0)
    a1, a2, a3 = mk(A, d1), mk(A, d2), mk(A3, d3)
    fp8._lib.fp8_mm(ctypes.byref(a1), torch.cuda.current_stream().cuda_stream)
    fp8.fp8_mm_batched(a2, 1, 0, 0, 0)
    fp8.fp8_mm_batched(a3, 3, m * lda, 0, m * n)
    torch.cuda.synchronize()
    assert torch.equal(d1.view(torch.int16), d2.view(torch.int16))
    for bi in range(3):
        # batched launches pick their tile configuration on batch x tiles, so
        # compare within the GEMM tolerance rather than bit for bit
        assert torch.equal(d3[bi].view(torch.int16), d3[0].view(torch.int16))


@pytest.mark.parametrize("batch,m,n,k,a_major,b_major", [(64, 512, 512, 512, 0, 0), (8, 1024, 2048, 1024, 0, 1),
                                                         (4, 2048, 1024, 4096, 1, 1)])
def test_mm_batched_large_sampled(fp8, batch, m, n, k, a_major, b_major):
    """The pages' bmm shapes (64 x 512^3, 8 x 1024 x 2048) and a dW-like batch."""
    rng = np.random.default_rng(batch + m + k)
    run_batched(fp8, rng, batch, m, n, k, a_major, b_major, full=False)


# ---------------------------------------------------------------- stream-K

SK = 8                         # FP8_TILE_STREAMK
SK_TILES = [1 | SK, 2 | SK, 3 | SK]    # 128x128, 128x256 and 256x256 pair tiles with stream-K forced
SK_FLAG_BYTES = 160 * 8 * 4    # the workspace's zero-at-rest flag block


def flags_clear(ws):
    return int(ws[:SK_FLAG_BYTES].view(torch.int32).abs().sum().item()) == 0


@pytest.mark.parametrize("tile", SK_TILES)
@pytest.mark.parametrize("a_major,b_major", LAYOUTS)
@pytest.mark.parametrize("m,n,k", [(256, 384, 2048), (300, 200, 1000), (64, 192, 640), (3, 100, 1100)])
def test_mm_stream_k_full(fp8, a_major, b_major, m, n, k, tile):
    """Stream-K forced on few-tile, long-K shapes (every tile cut between 2 to
    ~6 CTAs; ragged rows, columns and k): full comparison with the oracle, and
    every flag of the workspace back at zero after the launch."""
    rng = np.random.default_rng(m + n + k + tile)
    ws = fp8.mm_workspace(m, n, k, "cuda")
    run_case(fp8, rng, m, n, k, a_major, b_major, full=True, tile=tile, workspace=ws)
    assert flags_clear(ws)


@pytest.mark.parametrize("tile", [0] + SK_TILES)
@pytest.mark.parametrize("m,n,k,a_major,b_major", [
    (2048, 1536, 6912, 0, 0), (2048, 1536, 6912, 0, 1), (1536, 1536, 2048, 1, 1),
    (4096, 4096, 384, 0, 0), (512, 6912, 1536, 1, 1)])
def test_mm_stream_k_large_sampled(fp8, m, n, k, a_major, b_major, tile):
    """Production-sized shapes with a workspace: AUTO (which picks stream-K
    where the cost model says it pays) and forced stream-K, including the
    hybrid schedule (4096 x 4096 tiles: whole waves data-parallel, the last
    ones stream-K), against sampled oracle outputs; the fp8 bias rides on the
    finishing CTA's epilogue."""
    rng = np.random.default_rng(m + k + tile)
    ws = fp8.mm_workspace(m, n, k, "cuda")
    run_case(fp8, rng, m, n, k, a_major, b_major, full=False, tile=tile, workspace=ws, bias_kind="e4m3")
    assert flags_clear(ws)


@pytest.mark.parametrize("tile", SK_TILES)
def test_mm_stream_k_deterministic_and_reusable(fp8, tile):
    """The finishing CTA adds the partials in CTA order: two launches reusing
    one workspace give the same bits."""
    m, n, k = 700, 520, 3000
    rng = np.random.default_rng(5)
    ws = fp8.mm_workspace(m, n, k, "cuda")
    _, y1, _ = run_case(fp8, rng, m, n, k, 0, 1, full=False, tile=tile, workspace=ws)
    rng = np.random.default_rng(5)
    _, y2, _ = run_case(fp8, rng, m, n, k, 0, 1, full=False, tile=tile, workspace=ws)
    assert np.array_equal(y1, y2) and flags_clear(ws)


def test_mm_stream_k_needs_workspace(fp8):
    """Forced stream-K without (or with too small) a workspace is refused
    before anything is enqueued; AUTO without one simply runs data-parallel."""
    m, n, k = 256, 256, 1024
    A = torch.zeros((m, k), dtype=torch.uint8, device="cuda")
    B = torch.zeros((n, k), dtype=torch.uint8, device="cuda")
    sc = torch.ones(2, device="cuda")
    d = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    small = torch.zeros(SK_FLAG_BYTES, dtype=torch.uint8, device="cuda")
    for ws in (None, small):
        args = fp8.MmArgs(m, n, k, A.data_ptr(), 0, 0, k, B.data_ptr(), 0, 0, k, sc.data_ptr(), sc.data_ptr() + 4,
                          None, 0, None, d.data_ptr(), n, 1 | SK,
                          ws.data_ptr() if ws is not None else None, ws.numel() if ws is not None else 0)
        assert fp8._lib.fp8_mm(ctypes.byref(args), torch.cuda.current_stream().cuda_stream) == fp8.FP8_ERR_WORKSPACE
    assert fp8._lib.fp8_mm(ctypes.byref(fp8.MmArgs(m, n, k, A.data_ptr(), 0, 0, k, B.data_ptr(), 0, 0, k,
                                                   sc.data_ptr(), sc.data_ptr() + 4, None, 0, None, d.data_ptr(),
                                                   n, 0)), torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert torch.all(d.float() == 0) and fp8.fp8_get_device_status() == 0


@pytest.mark.parametrize("tile", [0] + SK_TILES)
def test_mm_pair_stream_k(fp8, tile):
    """dX and dW of one linear in one launch with stream-K over both problems'
    k-blocks (unequal k: 520 vs 2100), against the oracle."""
    rng = np.random.default_rng(41)
    M, N, K = 2100, 520, 300
    g8 = codes_like_tensor(rng, 1, (M, N), 3000.0)
    w8 = codes_like_tensor(rng, 0, (N, K), 60.0)
    x8 = codes_like_tensor(rng, 0, (M, K), 60.0)
    gs, ldg = store(g8, 0, 0)
    wst, ldw = store(w8, 0, 0)
    xs, ldx = store(x8, 0, 0)
    G, W, X = (torch.from_numpy(t).cuda() for t in (gs, wst, xs))
    sc = torch.tensor([3.0, 0.5, 0.25], device="cuda")
    dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dw = torch.empty(N, K, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(max(fp8.fp8_mm_workspace_bytes(M, K, N), fp8.fp8_mm_workspace_bytes(N, K, M)),
                     dtype=torch.uint8, device="cuda")
    p = lambda t: t.data_ptr()  # noqa: E731
    s4 = sc.data_ptr()
    a = fp8.MmArgs(M, K, N, p(G), 1, 0, ldg, p(W), 0, 1, ldw, s4, s4 + 4, None, 0, None, p(dx), K, tile,
                   p(ws), ws.numel())
    b = fp8.MmArgs(N, K, M, p(G), 1, 1, ldg, p(X), 0, 1, ldx, s4, s4 + 8, None, 0, None, p(dw), K, tile)
    fp8.fp8_mm_pair(a, b)
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0 and flags_clear(ws)
    gemm_dx, _, sab = oracle.gemm_acc(gs, 1, ldg, 1, wst, 0, 1, ldw, M, K, N)
    want, _ = oracle.epilogue(gemm_dx, 3.0, 0.5)
    assert_gemm_close(dx.cpu().view(torch.int16).numpy().view(np.uint16), want, sab, 3.0, 0.5, "pair sk dx")
    gemm_dw, _, sab = oracle.gemm_acc(gs, 1, 1, ldg, xs, 0, 1, ldx, N, K, M)
    want, _ = oracle.epilogue(gemm_dw, 3.0, 0.25)
    assert_gemm_close(dw.cpu().view(torch.int16).numpy().view(np.uint16), want, sab, 3.0, 0.25, "pair sk dw")


@pytest.mark.parametrize("a_major,b_major", LAYOUTS)
def test_mm_nan_codes_propagate(fp8, a_major, b_major):
    """NaN codes in the operands (E4M3 0x7F/0xFF in A, E5M2 0x7E in B): every
    output whose dot product contains one is NaN, all others are finite and
    match the oracle."""
    rng = np.random.default_rng(77 + 2 * a_major + b_major)
    m, n, k = 300, 260, 200
    A = codes_like_tensor(rng, 0, (m, k), 60.0)
    B = codes_like_tensor(rng, 1, (n, k), 3000.0)
    A[11, 3], A[250, 199] = 0x7F, 0xFF
    B[100, 0] = 0x7E
    _, y, _ = run_case(fp8, rng, m, n, k, a_major, b_major, fmt_a=0, fmt_b=1, a_codes=A, b_codes=B)
    yf = oracle.bf16_to_f32(y)
    nan_rows, nan_cols = {11, 250}, {100}
    for i in range(m):
        for_rows = np.isnan(yf[i])
        if i in nan_rows:
            assert for_rows.all()
        else:
            assert np.array_equal(np.where(for_rows)[0], np.array(sorted(nan_cols)))


@pytest.mark.parametrize("a_major,b_major", LAYOUTS)
def test_mm_inf_codes_follow_ieee(fp8, a_major, b_major):
    """E5M2 infinities in A against E4M3 B: outputs are what IEEE fp32
    accumulation gives, as in the oracle -- +-inf for one infinite product,
    NaN for inf x 0 and for products of both infinite signs -- and bf16 +-inf
    / NaN after the epilogue; all other outputs finite and within tolerance."""
    rng = np.random.default_rng(91 + 2 * a_major + b_major)
    m, n, k = 260, 200, 150
    A = codes_like_tensor(rng, 1, (m, k), 3000.0)
    B = codes_like_tensor(rng, 0, (n, k), 60.0)
    B[B == 0x80] = 0x08
    B[B == 0x00] = 0x08
    A[5, 10] = 0x7C                      # row 5: +-inf by the sign of B(j, 10)
    A[77, 149] = 0xFC                    # row 77: -+inf
    A[130, 3] = 0x7C
    B[60, 3] = 0x00                      # (130, 60): inf x 0 = NaN; rest of row 130 inf
    A[200, 20], A[200, 21] = 0x7C, 0xFC
    B[:, 20] = B[:, 21] = 0x38           # row 200: +inf - inf = NaN everywhere
    _, y, want = run_case(fp8, rng, m, n, k, a_major, b_major, fmt_a=1, fmt_b=0, a_codes=A, b_codes=B)
    yf, wf = oracle.bf16_to_f32(y), oracle.bf16_to_f32(want)
    assert np.isinf(yf[5]).all() and np.isinf(yf[77]).all() and np.isnan(yf[200]).all()
    assert np.isnan(yf[130, 60]) and np.isinf(yf[130, :60]).all()
    assert np.array_equal(np.isnan(yf), np.isnan(wf)) and np.array_equal(yf[np.isinf(wf)], wf[np.isinf(wf)])
    assert np.isfinite(np.delete(yf, [5, 77, 130, 200], axis=0)).all()
