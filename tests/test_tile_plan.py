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
