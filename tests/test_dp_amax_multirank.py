"""The data-parallel amax exchange (fp8_delayed_scaling_03_b200.dp) with two
gloo ranks on CPU: one MAX all-reduce over the rings' pending-amax words gives
every rank the global amax -- including 0, inf and subnormal amaxes, where the
integer MAX of the bits must still be the float max -- and the ring step the
oracle takes with it is identical on both ranks."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

# per ring: (rank 0 local amax, rank 1 local amax), three steps
AMAX = [
    [(1.5, 3.25), (np.inf, 2.0), (0.0, 0.0), (7e-39, 1e-38)],
    [(40.0, 0.5), (1.0, 1.0), (0.0, 6.0), (448.0, 447.0)],
    [(0.25, 0.125), (3.0, np.inf), (2.0, 0.0), (1e-30, 1e-20)],
]


class _CpuRing:
    """The ring interface dp.py uses (buf, H, words) on a host buffer."""

    def __init__(self, H):
        self.H = H
        self.buf = torch.zeros(H + 4, dtype=torch.float32)
        self.buf[H] = 1.0

    def words(self):
        return self.buf.view(torch.int32)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import oracle
    from fp8_delayed_scaling_03_b200 import dp
    H = 16
    rings = [_CpuRing(H) for _ in AMAX[0]]
    orings = [oracle.Ring(H) for _ in AMAX[0]]
    res = []
    for step in AMAX:
        for r, (a0, a1) in zip(rings, step):
            dp.scratch_word(r).copy_(torch.tensor([(a0, a1)[rank]], dtype=torch.float32).view(torch.int32))
        dp.allreduce_pending_amax(rings)
        got = [float(dp.scratch_word(r).view(torch.float32).item()) for r in rings]
        for r, o, a in zip(rings, orings, got):  # the ring step, as fp8_ring_finalize takes it
            o.advance(np.float32(a), oracle.E4M3)
            r.buf.zero_()
        res.append((got, [(float(o.scale), o.step, o.hist.tolist()) for o in orings]))
    out[rank] = res
    dist.barrier()
    dist.destroy_process_group()


def test_dp_amax_allreduce_gloo_world2():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1], "both ranks must hold the same amaxes and ring states"
    for (got, _), step in zip(res[0], AMAX):
        want = [float(np.float32(max(a0, a1))) for a0, a1 in step]
        assert got == want, (got, want)
