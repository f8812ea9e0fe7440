"""The benchmark step's two schedules give the same results bit for bit: the
weights quantized inside each fp8_linear_forward (with x, one launch), or on a
second stream ahead of the forward linears, which then take them
pre-quantized with the quantize's snapshot as their scale.  Outputs (y, dX,
dW, dbias), the fp8 copies, the snapshots and every ring word must match
after two steps, captured as CUDA graphs as bench.py times them."""
import pytest
import torch

import bench
import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


SHAPES = (wl.LinearShape("a", 300, 256, 640), wl.LinearShape("b", 300, 640, 200), wl.LinearShape("c", 300, 200, 256))


def build(F, bias):
    return [bench.Linear(F, s, 9100 + 10 * j, torch.device("cuda"), bias=bias, outliers=(j == 0))
            for j, s in enumerate(SHAPES)]


def state(L):
    out = [L.y, L.dx, L.dw, L.x8, L.w8, L.g8, L.sc[:6], L.rings.view(torch.int32)]
    if L.db is not None:
        out.append(L.db)
    return [t.clone() for t in out]


@pytest.mark.parametrize("bias", [bench.BIAS_NONE, bench.BIAS_BF16, bench.BIAS_E4M3])
def test_side_stream_weights_match_fused(fp8, bias):
    results = []
    for side_mode in (False, True):
        lins = build(fp8, bias)
        stream = torch.cuda.Stream()
        side = torch.cuda.Stream() if side_mode else None
        graph = bench.capture_step(fp8, lins, stream, 1, side)   # eager step + captured step replayed once
        torch.cuda.synchronize()
        assert fp8.fp8_get_device_status() == 0
        results.append([state(L) for L in lins])
        del graph
    for j, (a, b) in enumerate(zip(*results)):
        for i, (ta, tb) in enumerate(zip(a, b)):
            assert torch.equal(ta.view(torch.uint8), tb.view(torch.uint8)), (SHAPES[j].name, i)
