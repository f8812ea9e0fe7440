"""Sizes past 2^31 elements on the GPU: the quantize's chunk indices, amax
reduction and ring step, and the GEMM's output addressing (TMA-stored tiles
and the element-store path of an unaligned row pitch) must not wrap at 32
bits.  Outputs are checked at seeded sample points (plus every planted value
and the tensor's last elements) against the oracle; the amax is fixed by
construction (a planted maximum at the very last element)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_codes_equal, assert_gemm_close, oracle_ring_words, ring_words

pytestmark = pytest.mark.gpu

E31 = 2 ** 31


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def test_quantize_past_2_31_elements(fp8):
    rows, cols = 32768, 65552                     # 2,148,007,936 elements, bf16 (4.3 GB)
    n = rows * cols
    assert n > E31
    g = torch.Generator(device="cuda")
    g.manual_seed(20261203)
    x = torch.randn(rows, cols, device="cuda", dtype=torch.bfloat16, generator=g).clamp_(-100.0, 100.0)
    flat = x.view(-1)
    plant = {E31 - 1: 37.5, E31: -61.25, E31 + 1: 0.0078125, E31 + 17: -99.5, n - 1: 1000.0}
    for i, v in plant.items():
        flat[i] = v
    fmt = fp8.FP8_E4M3
    ring = fp8.ScaleRing(16, seed_amax=250.0, fmt=fmt)
    oring = oracle.Ring(16)
    oring.seed(250.0, fmt)
    out = torch.full((rows, cols), 0xA5, dtype=torch.uint8, device="cuda")
    amax = torch.full((1,), -1.0, device="cuda")
    scale = torch.full((1,), -1.0, device="cuda")
    fp8.fp8_quantize(x, fmt, ring.buf, 16, out, amax, scale)
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0
    s = np.float32(oring.scale)
    assert np.float32(scale.item()) == s
    assert np.float32(amax.item()) == np.float32(1000.0)
    oring.advance(1000.0, fmt)
    assert np.array_equal(ring_words(ring), oracle_ring_words(oring))
    rng = np.random.default_rng(31)
    idx = np.concatenate([rng.integers(0, n, 300_000), np.array(sorted(plant), np.int64),
                          np.arange(E31 - 4096, E31 + 4096), np.arange(n - 8192, n)]).astype(np.int64)
    it = torch.from_numpy(idx).cuda()
    xs = flat[it].cpu().view(torch.int16).numpy().view(np.uint16).reshape(1, -1)
    got = out.view(-1)[it].cpu().numpy().reshape(1, -1)
    want = oracle.quantize_codes(xs, oracle.DT_BF16, fmt, s)
    assert_codes_equal(got, want, fmt)
    del x, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("n,ldd", [(32784, 32784), (32772, 32772)])
def test_mm_output_past_2_31_elements(fp8, n, ldd):
    """65536 x n x 160 with a 4.3 GB bf16 output: TMA-stored tiles (row pitch a
    multiple of 16 bytes) and the element-store path (pitch 65544 bytes)."""
    m, k = 65536, 160
    assert m * ldd > E31
    rng = np.random.default_rng(n)
    A = oracle.encode(0, (rng.standard_normal((m, k)) * 60).astype(np.float32))
    B = oracle.encode(0, (rng.standard_normal((n, k)) * 60).astype(np.float32))
    lda = ldb = (k + 15) // 16 * 16
    a_st = np.zeros((m, lda), np.uint8)
    a_st[:, :k] = A
    b_st = np.zeros((n, ldb), np.uint8)
    b_st[:, :k] = B
    sa, sb = 2.0, 0.5
    sc = torch.tensor([sa, sb], dtype=torch.float32, device="cuda")
    d = torch.full((m, ldd), float("nan"), dtype=torch.bfloat16, device="cuda")
    fp8.fp8_mm(m, n, k, torch.from_numpy(a_st).cuda(), 0, 0, lda, torch.from_numpy(b_st).cuda(), 0, 0, ldb,
               sc[0:1], sc[1:2], d, ldd)
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0
    assert not bool(torch.isnan(d[:, :n]).any()), "every output element is written"
    pi = np.concatenate([rng.integers(0, m, 200_000), np.full(n, m - 1), np.arange(m - 256, m).repeat(4)])
    pj = np.concatenate([rng.integers(0, n, 200_000), np.arange(n), np.tile([0, 1, n - 2, n - 1], 256)])
    pi, pj = pi.astype(np.int64), pj.astype(np.int64)
    got = d[torch.from_numpy(pi).cuda(), torch.from_numpy(pj).cuda()].cpu().view(torch.int16).numpy().view(np.uint16)
    acc, sab = oracle.gemm_acc_points(pi, pj, a_st, 0, lda, 1, b_st, 0, ldb, 1, k)
    want, _ = oracle.epilogue(acc, sa, sb)
    assert_gemm_close(got, want, sab, sa, sb, f"mm {m}x{n}x{k} ldd {ldd}")
    del d
    torch.cuda.empty_cache()
