"""The GEMM tile choice (fp8_mm_plan: what fp8_mm / fp8_mm_pair would launch),
host arithmetic only, on a 148-SM B200.  These pin the cost model's decisions
that were measured on the GPU: 256x256 CTA-pair tiles once a launch runs more
than three rounds of tiles (8192^3 at 3.2 PFLOP/s vs 2.8 on 128x256;
4096^3 50 vs 53 us), 128x256 for two- and three-round launches (2048 x 6912 x
1536: 20.0 vs 20.8 us), 128x128 where 128x256 would leave SMs idle
(2048 x 1024 x 1024: 6.1 vs 6.7 us), and the LPT-scheduled 128x128 dX+dW
launch of a 1024 x 1024 linear at M = 2048."""
import pytest

A = 0x100000  # fake 16-byte aligned device addresses; nothing is dereferenced


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def args(F, m, n, k, a_major=0, b_major=0, tile_cfg=0):
    lda = k if a_major == F.FP8_K_MAJOR else m
    ldb = k if b_major == F.FP8_K_MAJOR else n
    lda, ldb = (lda + 15) // 16 * 16, (ldb + 15) // 16 * 16
    return F.MmArgs(m, n, k, A, 0, a_major, lda, A + 0x10000, 0, b_major, ldb, A + 0x20000, A + 0x20010,
                    None, 0, None, A + 0x30000, n, tile_cfg)


@pytest.mark.parametrize("m,n,k,cfg,tiles,units", [
    (8192, 8192, 8192, 3, 1024, 74),      # 14 rounds of pair tiles
    (4096, 4096, 4096, 3, 256, 74),       # 4 rounds
    (4096, 11008, 4096, 3, 688, 74),
    (2048, 6912, 1536, 2, 432, 148),      # 3 rounds of 128x256
    (2048, 4096, 1024, 2, 256, 148),
    (2048, 1024, 1024, 1, 128, 128),      # 128x256 would use 64 SMs
    (2048, 1024, 4096, 1, 128, 128),
])
def test_single_problem_choice(fp8, m, n, k, cfg, tiles, units):
    p = fp8.fp8_mm_plan(args(fp8, m, n, k))
    assert (p.tile_cfg, p.tiles, p.units) == (cfg, tiles, units)
    assert p.est_us > 0


def test_dx_dw_pair_of_a_1024_linear(fp8):
    F = fp8
    dx = args(F, 2048, 1024, 1024, F.FP8_K_MAJOR, F.FP8_MN_MAJOR)   # G8 . W8
    dw = args(F, 1024, 1024, 2048, F.FP8_MN_MAJOR, F.FP8_MN_MAJOR)  # G8^T . X8
    p = F.fp8_mm_plan(dx, dw)
    assert (p.tile_cfg, p.tiles, p.units) == (1, 128 + 64, 148)


def test_estimate_grows_with_k_and_forced_configs_echo(fp8):
    F = fp8
    est = [F.fp8_mm_plan(args(F, 2048, 2048, k)).est_us for k in (1024, 2048, 4096, 8192)]
    assert all(a < b for a, b in zip(est, est[1:]))
    for cfg in (1, 2, 3, 4):
        p = F.fp8_mm_plan(args(F, 2048, 2048, 2048, tile_cfg=cfg))
        assert p.tile_cfg == cfg and p.est_us == 0.0


def test_plan_validation(fp8):
    F = fp8
    assert F._lib.fp8_mm_plan(None, None, 148, None) == F.FP8_ERR_INVALID_ARG
    info = F.MmPlanInfo()
    import ctypes
    a = args(F, 256, 256, 256)
    assert F._lib.fp8_mm_plan(ctypes.byref(a), None, 0, ctypes.byref(info)) == F.FP8_ERR_INVALID_ARG
    bad = args(F, 256, 256, 256)
    bad.lda = 264                                       # not a multiple of 16
    assert F._lib.fp8_mm_plan(ctypes.byref(bad), None, 148, ctypes.byref(info)) == F.FP8_ERR_MISALIGNED
    empty = F.fp8_mm_plan(args(F, 0, 256, 256))
    assert (empty.tile_cfg, empty.tiles, empty.units) == (0, 0, 0)
    one = F.fp8_mm_plan(args(F, 0, 256, 256), args(F, 256, 256, 256))   # the empty problem is dropped
    assert one.tiles == 4 and one.tile_cfg == 1


WS = 0x8000000  # fake workspace address


def with_ws(F, a, nbytes=None):
    a.workspace = WS
    a.workspace_bytes = F.fp8_mm_workspace_bytes(a.m, a.n, a.k) if nbytes is None else nbytes
    return a


def test_workspace_bytes(fp8):
    F = fp8
    flags, slot = 160 * 8 * 4, 128 * 256 * 4
    assert F.fp8_mm_workspace_bytes(0, 10, 10) == 0 and F.fp8_mm_workspace_bytes(10, 10, 0) == 0
    assert F.fp8_mm_workspace_bytes(64, 192, 128) == flags + 2 * slot     # two 128 x 128 x 128 blocks
    assert F.fp8_mm_workspace_bytes(2048, 1536, 6912) == flags + 160 * slot
    # the linear backward's workspace is its bias-gradient scratch only
    assert F.fp8_linear_workspace_bytes(2048, 1536, 6912) >= F.fp8_dbias_workspace_bytes(2048, 1536)


@pytest.mark.parametrize("m,n,k,a_major,b_major", [
    (2048, 1536, 6912, 0, 1),     # dX with contraction 6912: 96 tiles of 128x256 on 148 SMs
    (2048, 1536, 6912, 0, 0),     # forward with K = 6912
    (512, 1536, 6912, 0, 1),
    (4096, 11008, 4096, 0, 0),
])
def test_auto_never_stream_k(fp8, m, n, k, a_major, b_major):
    """AUTO stays data-parallel even with a workspace (measured on a B200: the
    stream-K plans the cost model picked were slower inside the benchmark
    steps); forced stream-K still plans its ranges."""
    F = fp8
    plain = F.fp8_mm_plan(args(F, m, n, k, a_major, b_major))
    ws = F.fp8_mm_plan(with_ws(F, args(F, m, n, k, a_major, b_major)))
    assert plain.stream_k_ctas == 0 and ws.stream_k_ctas == 0
    assert (ws.tile_cfg, ws.tiles, ws.units, ws.est_us) == (plain.tile_cfg, plain.tiles, plain.units, plain.est_us)
    forced = F.fp8_mm_plan(with_ws(F, args(F, m, n, k, a_major, b_major, tile_cfg=2 | F.FP8_TILE_STREAMK)))
    assert forced.stream_k_ctas > 0 and forced.tile_cfg == 2 | F.FP8_TILE_STREAMK


def test_stream_k_forced_and_hybrid(fp8):
    F = fp8
    p = F.fp8_mm_plan(with_ws(F, args(F, 4096, 4096, 384, tile_cfg=1 | F.FP8_TILE_STREAMK)))
    # 1024 tiles of 128x128: five whole waves of 148 data-parallel, 284 tiles' k-blocks stream-K
    assert p.tile_cfg == 1 | F.FP8_TILE_STREAMK and p.dp_tiles == 5 * 148 and p.stream_k_ctas == 148
    import ctypes
    info = F.MmPlanInfo()
    a = with_ws(F, args(F, 256, 256, 1024, tile_cfg=1 | F.FP8_TILE_STREAMK), nbytes=0)
    a.workspace = None
    assert F._lib.fp8_mm_plan(ctypes.byref(a), None, 148, ctypes.byref(info)) == F.FP8_ERR_WORKSPACE
    bad = args(F, 256, 256, 1024, tile_cfg=4 | F.FP8_TILE_STREAMK)      # split-K has no stream-K
    assert F._lib.fp8_mm_plan(ctypes.byref(bad), None, 148, ctypes.byref(info)) == F.FP8_ERR_INVALID_ARG
    pair = F.fp8_mm_plan(with_ws(F, args(F, 4096, 11008, 4096, tile_cfg=3 | F.FP8_TILE_STREAMK)))
    # 688 pair tiles on 74 pairs: eight whole waves, the rest stream-K over the 74 pairs
    assert pair.dp_tiles == 8 * 74 and pair.stream_k_ctas == 74 and pair.units == 74
    mis = with_ws(F, args(F, 256, 256, 1024))
    mis.workspace = WS + 8                                              # not 16-byte aligned
    assert F._lib.fp8_mm_plan(ctypes.byref(mis), None, 148, ctypes.byref(info)) == F.FP8_ERR_WORKSPACE
