"""Data-parallel delayed scaling: the one exchange the method needs across
data-parallel replicas.  Every rank's ring must take the same step, so the
amax of a launch is all-reduced with MAX before the ring step (a per-tensor
max over all ranks' shards is the amax of the whole global batch).

Per step on each rank, stream-ordered, no host synchronization:

    fp8_quantize_ex(args, FP8_QUANTIZE_DEFER_RING_STEP)  # cast with the ring's scale;
                                                         # local amax -> ring scratch word
    ... the GEMMs (the all-reduce may overlap them: the cast did not need it) ...
    allreduce_pending_amax(rings, group)                 # ONE MAX all-reduce over all rings
    finalize_rings(rings, fmts)                          # the ring step with the global amax

The scratch word is 32-bit word H + 3 of a ring.  Amaxes are non-negative
floats (NaN never enters them), whose IEEE bit patterns order like the values,
so a 32-bit integer MAX of the bits is the float max, exactly.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def scratch_word(ring) -> torch.Tensor:
    """int32 view (one element) of a ring's pending-amax word."""
    return ring.words()[ring.H + 3: ring.H + 4]


def allreduce_pending_amax(rings, group=None) -> None:
    """All-reduce MAX of the pending amax of every ring in one collective."""
    if not rings:
        return
    words = torch.cat([scratch_word(r) for r in rings])
    dist.all_reduce(words, op=dist.ReduceOp.MAX, group=group)
    for r, w in zip(rings, words):
        scratch_word(r).copy_(w.view(1))


def finalize_rings(rings, fmts, amax_outs=None) -> None:
    """fp8_ring_finalize on each ring (device rings only)."""
    from . import fp8_ring_finalize
    for i, (r, f) in enumerate(zip(rings, fmts)):
        fp8_ring_finalize(r.buf, r.H, f, amax_outs[i] if amax_outs is not None else None)
