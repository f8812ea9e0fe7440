"""GPU side of the data-parallel amax exchange: fp8_quantize_ex with
FP8_QUANTIZE_DEFER_RING_STEP casts with the ring's scale and leaves only the
local amax in the ring's scratch word; after a MAX over the ranks' words,
fp8_ring_finalize takes the ring step the oracle takes with the global amax.
Two ranks are emulated on one GPU (the MAX done by a device op), and a real
one-rank NCCL group runs the collective path of dp.allreduce_pending_amax."""
import socket

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from helpers import assert_codes_equal, bits, fp8_buffer, host_rows, oracle_ring_words, ring_words

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def test_deferred_step_two_ranks_emulated(fp8):
    from fp8_delayed_scaling_03_b200 import dp
    H = 16
    rings = [fp8.ScaleRing(H), fp8.ScaleRing(H)]
    orng = oracle.Ring(H)
    for step in range(4):
        xs = [wl.normal((1000, 700), (1.0, 6.0)[r] * (1 + step), 1700 + 10 * step + r) for r in range(2)]
        xd = [x.cuda() for x in xs]
        outs = [fp8_buffer(1000, 700) for _ in range(2)]
        sc = torch.full((4,), -1.0, device="cuda")
        before = [ring_words(r) for r in rings]
        for r in range(2):
            a = fp8.quantize_args(xd[r], 0, rings[r].buf, H, outs[r], sc[2 * r:2 * r + 1], sc[2 * r + 1:2 * r + 2])
            fp8.fp8_quantize_ex(a, fp8.FP8_QUANTIZE_DEFER_RING_STEP)
        torch.cuda.synchronize()
        amaxes = [oracle.amax(bits(x), oracle.DT_BF16) for x in xs]
        for r in range(2):
            w = ring_words(rings[r])
            # history, scale and step untouched; the local amax pending in the scratch word
            assert np.array_equal(w[:H + 3], before[r][:H + 3])
            assert np.uint32(w[H + 3]) == np.float32(amaxes[r]).view(np.uint32)
            assert sc[2 * r + 1].item() == orng.scale  # cast with the ring's (pre-step) scale
            assert sc[2 * r].item() == -1.0            # amax_out waits for the finalize
            q = oracle.quantize_codes(bits(xs[r]), oracle.DT_BF16, 0, orng.scale)
            assert_codes_equal(host_rows(outs[r]), q, 0)
        # the all-reduce, emulated: MAX of the two words into both
        m = torch.maximum(dp.scratch_word(rings[0]), dp.scratch_word(rings[1]))
        for r in rings:
            dp.scratch_word(r).copy_(m)
        amax_out = torch.full((2,), -1.0, device="cuda")
        dp.finalize_rings(rings, [0, 0], [amax_out[0:1], amax_out[1:2]])
        torch.cuda.synchronize()
        g = max(amaxes)
        orng.advance(g, oracle.E4M3)
        assert amax_out.tolist() == [g, g]
        for r in rings:
            assert np.array_equal(ring_words(r), oracle_ring_words(orng))
    assert fp8.fp8_get_device_status() == 0


def test_quantize_ex_without_flags_equals_quantize(fp8):
    H = 16
    r1, r2 = fp8.ScaleRing(H), fp8.ScaleRing(H)
    x = wl.normal((513, 1000), 3.0, 1750).cuda()
    o1, o2 = fp8_buffer(513, 1000), fp8_buffer(513, 1000)
    s1, s2 = torch.zeros(2, device="cuda"), torch.zeros(2, device="cuda")
    for _ in range(3):
        fp8.fp8_quantize(x, 0, r1.buf, H, o1, s1[0:1], s1[1:2])
        fp8.fp8_quantize_ex(fp8.quantize_args(x, 0, r2.buf, H, o2, s2[0:1], s2[1:2]), 0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    assert np.array_equal(ring_words(r1), ring_words(r2))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_dp_collective_one_rank_nccl(fp8):
    """dp.allreduce_pending_amax through a real NCCL group (one rank: the MAX
    is the identity) gives the same ring as the in-kernel last-block step."""
    import datetime

    import torch.distributed as dist
    from fp8_delayed_scaling_03_b200 import dp
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        H = 8
        rd, rr = [fp8.ScaleRing(H), fp8.ScaleRing(H)], [fp8.ScaleRing(H), fp8.ScaleRing(H)]
        for step in range(3):
            xs = [wl.normal((300, 260), 2.0 ** (step + i), 1760 + step + 5 * i).cuda() for i in range(2)]
            od = [fp8_buffer(300, 260) for _ in range(2)]
            orr = [fp8_buffer(300, 260) for _ in range(2)]
            for i in range(2):
                fp8.fp8_quantize_ex(fp8.quantize_args(xs[i], i, rd[i].buf, H, od[i]), fp8.FP8_QUANTIZE_DEFER_RING_STEP)
                fp8.fp8_quantize(xs[i], i, rr[i].buf, H, orr[i])
            dp.allreduce_pending_amax(rd)
            dp.finalize_rings(rd, [0, 1])
            torch.cuda.synchronize()
            for i in range(2):
                assert torch.equal(od[i], orr[i])
                assert np.array_equal(ring_words(rd[i]), ring_words(rr[i]))
    finally:
        dist.destroy_process_group()
