"""The benchmarked step itself against the oracle, at full size: the headline
workload's three M=4096 linears ({4096x11008, 11008x4096, 4096x4096}, x with
outliers), the production workload's six linears (M in {512, 2048}, E4M3
bias with its own scale, bias gradient) and the dim1024 training step's 72
linears (bf16 bias and bias gradient) are built, captured and replayed
exactly as bench.py times them (an eager step, then the captured graph
replayed once), and after those two steps every quantized byte (x8, w8, g8),
every scale snapshot and amax, and every ring word is compared with the
oracle's two steps bit for bit; y, dX and dW at sampled points (full rows,
full columns, random points) and dbias in full are compared within the GEMM
tolerance."""
import numpy as np
import pytest
import torch

import bench
import oracle
from helpers import assert_codes_equal, assert_gemm_close, bits, oracle_ring_words, sample_points

pytestmark = pytest.mark.gpu
E4, E5 = oracle.E4M3, oracle.E5M2


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def host_bits(t):
    return bits(t.detach().cpu())


@pytest.mark.parametrize("workload", ["c4", "c3", "dim1024"])
def test_benchmarked_step_matches_oracle(fp8, workload):
    device = torch.device("cuda")
    lins = bench.build_model(fp8, device, 0, workload)
    stream = torch.cuda.Stream()
    graph = bench.capture_step(fp8, lins, stream, 1)  # the eager step + one replay of the captured step
    torch.cuda.synchronize()
    assert fp8.fp8_get_device_status() == 0
    rng = np.random.default_rng(2024)
    for li, L in enumerate(lins):
        M, K, N = L.shape.M, L.shape.K, L.shape.N
        ldk, ldn = L.x8.shape[1], L.g8.shape[1]
        xb, wb, gb = host_bits(L.x), host_bits(L.w), host_bits(L.g)
        rx, rw, rg = (oracle.Ring(16) for _ in range(3))
        # step 1 (the same inputs): only its amaxes reach step 2, through the rings
        for t, r, f in ((xb, rx, E4), (wb, rw, E4), (gb, rg, E5)):
            r.advance(oracle.amax(t, oracle.DT_BF16), f)
        x8, ax, sx = oracle.quantize(xb, oracle.DT_BF16, E4, rx, ld_out=ldk)
        w8, aw, sw = oracle.quantize(wb, oracle.DT_BF16, E4, rw, ld_out=ldk)
        g8, ag, sg = oracle.quantize(gb, oracle.DT_BF16, E5, rg, ld_out=ldn)
        what = f"{workload} linear {li} ({M}x{K}x{N})"
        assert_codes_equal(L.x8.cpu().numpy()[:, :K], x8[:, :K], E4)
        assert_codes_equal(L.w8.cpu().numpy()[:, :K], w8[:, :K], E4)
        assert_codes_equal(L.g8.cpu().numpy()[:, :N], g8[:, :N], E5)
        sc = L.sc.cpu().numpy()
        assert list(sc[:6]) == [sx, sw, sg, ax, aw, ag], what
        for r, o in zip(L.rings, (rx, rw, rg)):
            assert np.array_equal(r.detach().cpu().view(torch.int32).numpy().view(np.uint32),
                                  oracle_ring_words(o)), what
        # GEMMs at sampled points, from the oracle's (= the GPU's) quantized bytes
        bias, bias_dt, bsc = None, 0, 1.0
        if L.bias == bench.BIAS_E4M3:
            bias, bias_dt, bsc = L.b8.cpu().numpy()[0], oracle.DT_E4M3, float(sc[6])
        elif L.bias == bench.BIAS_BF16:
            bias, bias_dt = host_bits(L.b), oracle.DT_BF16
        for name, out, a, fa, a_s, b, fb, b_s, I, J, Kc, sa, sb, with_bias in (
                ("y", L.y, x8, E4, (ldk, 1), w8, E4, (ldk, 1), M, N, K, sx, sw, True),
                ("dx", L.dx, g8, E5, (ldn, 1), w8, E4, (1, ldk), M, K, N, sg, sw, False),
                ("dw", L.dw, g8, E5, (1, ldn), x8, E4, (1, ldk), N, K, M, sg, sx, False)):
            pi, pj = sample_points(rng, I, J, nrows=8, ncols=8, nrand=20000)
            acc, sab = oracle.gemm_acc_points(pi, pj, a, fa, *a_s, b, fb, *b_s, Kc)
            if with_bias and bias is not None:
                want, _ = oracle.epilogue(acc, sa, sb, bias, bias_dt, bsc, col_idx=pj)
            else:
                want, _ = oracle.epilogue(acc, sa, sb)
            got = host_bits(out)[pi, pj]
            assert_gemm_close(got, want, sab, sa, sb, f"{what} {name}")
        if L.db is not None:
            want, _, sa_db = oracle.dbias(gb, oracle.DT_BF16, M, N)
            g = oracle.bf16_to_f32(host_bits(L.db)).astype(np.float64)
            o = oracle.bf16_to_f32(want).astype(np.float64)
            assert np.all(np.abs(g - o) <= np.maximum(oracle.bf16_ulp(o), 2e-6 * sa_db)), what
    del graph
