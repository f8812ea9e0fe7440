#!/usr/bin/env python
"""Throughput of the FP8 linear layer with delayed scaling on B200.

One step = forward + backward of every linear of a workload through the C ABI
(fp8_linear_forward, then fp8_linear_backward in reverse order), replayed as
one CUDA graph: per linear, quantize x and w (E4M3, delayed-scaling rings),
the forward GEMM with fused dequant (+ bias), quantize g (E5M2, + bias
gradient), dX and dW.  The headline workload is the generic large shapes at
M = 4096 tokens: three linears {4096x11008, 11008x4096, 4096x4096} (K x N),
x ~ N(0,1) with 0.1% outliers x50, w ~ N(0, 1/sqrt(K)), g ~ N(0, 1e-3), no
bias.  The value is TFLOP/s of the three GEMMs (6 M N K per linear) over the
whole step.  Inputs are synthetic, seeded and resident in HBM; the step's
working set (about 1.6 GB) is far larger than L2.

Extra keys of the same JSON line: `roofline` (the GEMM class of the headline
step), `kernels` (per-class times), `steps` (the dim1024 training step of the
pages' 12L/dim1024/B4xT512 model with bf16 bias + dbias, and the production
24L/dim1536/ffn6912 linears at M in {512, 2048} with an E4M3 bias and dbias),
`targets` (fwd, dX and dW as single launches at the production and large
shapes, warm and cold L2, against the measured peak, the nominal peak and
each shape's own roofline; standalone quantize GB/s), `e2e` (the headline
step with host buffers), `cpu_baseline` (the oracle on a sample).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own replica of the step (weak
scaling, no collective on the data path); the time is the max over ranks.
`--impl reference` times the CPU oracle on a bounded sample of the same
workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "FP8 linear fwd/dX/dW TFLOP/s and % dense FP8 peak; quantize GB/s % HBM"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0          # nominal dense fp8 : bf16 tensor-core ratio (4.5 : 2.25 PFLOP/s)
NOMINAL_FP8_TFLOPS = 4500.0
REF_TOKENS = 16             # tokens of the headline linears per reference-arm step
CPU_SAMPLE_TOKENS = 128     # tokens of the headline linears for the cpu_baseline sample


# --------------------------------------------------------------------------- helpers

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def reduce_max(value: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (the process group is already up)."""
    if world <= 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / max_seconds


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread while
    the timed region runs (reads only; changes no setting)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x100: "display_clock_setting", 0x10: "sync_boost"}

    def __init__(self, device_index: int):
        self.ok = False
        self.samples, self.reasons = [], set()
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.err = repr(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def report(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- workload

BIAS_NONE, BIAS_BF16, BIAS_E4M3 = "none", "bf16", "e4m3"


class Linear:
    """Device buffers and prebuilt C-ABI argument structs of one FP8 linear.
    bias: BIAS_NONE, BIAS_BF16 (bf16 bias, bf16 dbias) or BIAS_E4M3 (the bias
    stored as E4M3 codes with its own scale, quantized once here by the
    library's current-scaling quantize; bf16 dbias)."""

    def __init__(self, F, shape, seed_base, device, H=wl.HIST_LEN, bias=BIAS_BF16, outliers=False):
        M, K, N = shape.M, shape.K, shape.N
        self.shape = shape
        self.bias = bias
        ldk, ldn = (K + 15) // 16 * 16, (N + 15) // 16 * 16
        if outliers:
            self.x = wl.normal_with_outliers_device((M, K), 1.0, seed_base + wl.OP_X, seed_base + wl.OP_MASK, device)
        else:
            self.x = wl.normal_device((M, K), 1.0, seed_base + wl.OP_X, device)
        self.w = wl.normal_device((N, K), wl.weight_std(K), seed_base + wl.OP_W, device)
        self.b = wl.normal_device((N,), wl.BENCH_BIAS_STD, seed_base + wl.OP_BIAS, device) if bias != BIAS_NONE \
            else None
        self.g = wl.normal_device((M, N), 1e-3, seed_base + wl.OP_G, device)
        self.x8 = torch.zeros((M, ldk), dtype=torch.uint8, device=device)
        self.w8 = torch.zeros((N, ldk), dtype=torch.uint8, device=device)
        self.g8 = torch.zeros((M, ldn), dtype=torch.uint8, device=device)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        self.dx = torch.empty((M, K), dtype=torch.bfloat16, device=device)
        self.dw = torch.empty((N, K), dtype=torch.bfloat16, device=device)
        self.db = torch.empty((N,), dtype=torch.bfloat16, device=device) if bias != BIAS_NONE else None
        words = F.fp8_ring_bytes(H) // 4
        self.rings = torch.empty((3, words), dtype=torch.float32, device=device)
        for i in range(3):
            F.fp8_ring_init(self.rings[i], H)
        # sx, sw, sg, amax_x, amax_w, amax_g, bias_scale, bias amax
        self.sc = torch.zeros(8, dtype=torch.float32, device=device)
        sc = self.sc.data_ptr()
        self.bias_ptr, self.bias_dtype, self.bias_scale_ptr = None, F.FP8_DT_BF16, None
        if bias == BIAS_BF16:
            self.bias_ptr = self.b.data_ptr()
        elif bias == BIAS_E4M3:
            self.b8 = torch.zeros((1, ldn), dtype=torch.uint8, device=device)
            F.fp8_quantize(self.b.view(1, N), F.FP8_E4M3, None, 0, self.b8[:, :N], self.sc[7:8], self.sc[6:7])
            self.bias_ptr, self.bias_dtype, self.bias_scale_ptr = self.b8.data_ptr(), F.FP8_DT_E4M3, sc + 24
        need_dbias = bias != BIAS_NONE
        self.ws = torch.zeros(max(16, F.fp8_linear_workspace_bytes(M, N, K)), dtype=torch.uint8, device=device)
        p = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
        self.fwd = F.LinearFwdArgs(M, N, K, p(self.x), F.FP8_DT_BF16, K, None, p(self.w), F.FP8_DT_BF16, K, None,
                                   self.bias_ptr, self.bias_dtype, self.bias_scale_ptr, F.FP8_E4M3, F.FP8_E4M3, H,
                                   p(self.rings[0]), p(self.rings[1]), p(self.x8), ldk, p(self.w8), ldk,
                                   sc, sc + 4, sc + 12, sc + 16, p(self.y), N)
        # The weight quantized ahead of the forward (its own launch, its ring
        # stepping there), and the forward taking that pre-quantized weight
        # with its snapshot as the scale: the same outputs and ring words.
        self.qw = F.QuantizeArgs(p(self.w), F.FP8_DT_BF16, N, K, K, F.FP8_E4M3, p(self.rings[1]), H, p(self.w8), ldk,
                                 sc + 16, sc + 4)
        self.fwd_w8 = F.LinearFwdArgs(M, N, K, p(self.x), F.FP8_DT_BF16, K, None, p(self.w8), F.FP8_DT_E4M3, ldk,
                                      sc + 4, self.bias_ptr, self.bias_dtype, self.bias_scale_ptr, F.FP8_E4M3,
                                      F.FP8_E4M3, H, p(self.rings[0]), None, p(self.x8), ldk, None, 0,
                                      sc, sc + 4, sc + 12, None, p(self.y), N)
        self.w_ready = torch.cuda.Event()
        self.bwd = F.LinearBwdArgs(M, N, K, p(self.g), F.FP8_DT_BF16, N, None, F.FP8_E5M2, H, p(self.rings[2]),
                                   p(self.g8), ldn, sc + 8, sc + 20, p(self.x8), ldk, sc, F.FP8_E4M3,
                                   p(self.w8), ldk, sc + 4, F.FP8_E4M3, 1, 1, int(need_dbias), p(self.dx), K,
                                   p(self.dw), K, p(self.db), p(self.ws), self.ws.numel())

    def inputs(self):
        return [t for t in (self.x, self.w, self.b, self.g) if t is not None]

    def outputs(self):
        return [t for t in (self.y, self.dx, self.dw, self.db) if t is not None]


# Workloads: (description, builder).  Each builder returns the step's linears.
def _c4_linears(F, device, rank):
    return [Linear(F, s, wl.seed_for(4, 0, 0, extra=1 + rank * 1000 + j) * 10, device, bias=BIAS_NONE,
                   outliers=True) for j, s in enumerate(wl.C4_SHAPES)]


def _dim1024_linears(F, device, rank):
    lins = []
    for layer in range(wl.BENCH_LAYERS):
        for j, s in enumerate(wl.BENCH_LAYER):
            lins.append(Linear(F, s, wl.seed_for(2, 0, 0, extra=1 + rank * 1000 + layer * 10 + j) * 10, device))
    return lins


def _c3_linears(F, device, rank):
    return [Linear(F, s, wl.seed_for(3, 0, 0, extra=1 + rank * 1000 + j) * 10, device, bias=BIAS_E4M3)
            for j, s in enumerate(wl.C3_SHAPES)]


WORKLOADS = {
    "c4": ("generic large linears at M=4096 tokens: {4096x11008, 11008x4096, 4096x4096} (K x N), fwd+dX+dW, "
           "x ~ N(0,1) with 0.1% outliers x50, E4M3 x/w, E5M2 g, delayed scaling H=16, no bias",
           _c4_linears),
    "dim1024": ("12L/dim1024/B4xT512 linears: 12 layers x {q,k,v,o 1024x1024, up 1024x4096, down 4096x1024}, "
                "M=2048 tokens, fwd+dX+dW, E4M3 x/w, E5M2 g, delayed scaling H=16, bf16 bias + dbias",
                _dim1024_linears),
    "c3": ("production 24L/dim1536/ffn6912 linears: M in {512, 2048} x {1536x1536, 1536x6912, 6912x1536}, "
           "fwd+dX+dW, E4M3 x/w, E5M2 g, delayed scaling H=16, E4M3 bias with its own scale + dbias",
           _c3_linears),
}
HEADLINE = "c4"


def build_model(F, device, rank, workload=HEADLINE):
    return WORKLOADS[workload][1](F, device, rank)


def step_flops(lins) -> int:
    """fwd + dX + dW: 3 GEMMs of 2 M N K flops per linear."""
    return sum(6 * L.shape.M * L.shape.N * L.shape.K for L in lins)


def run_step(F, lins, stream, side=None):
    """Forward over the linears in order, then backward in reverse, through the
    C ABI.  With a side stream, the weights are quantized there first (one
    fp8_quantize per weight, in forward order) while the main stream runs the
    forward linears on the pre-quantized weights, each waiting only for its own
    weight: the weight casts overlap the earlier linears' GEMMs, which leave
    HBM mostly idle.  Weights do not depend on the activations, so this order
    is the step's own dependency graph."""
    lib = F._lib
    fwd, bwd = lib.fp8_linear_forward, lib.fp8_linear_backward
    h = stream.cuda_stream
    if side is None:
        for L in lins:
            s = fwd(ctypes.byref(L.fwd), h)
            if s:
                raise F.Fp8Error(s, "fp8_linear_forward")
    else:
        start = torch.cuda.Event()
        start.record(stream)
        side.wait_event(start)
        for L in lins:
            s = lib.fp8_quantize_ex(ctypes.byref(L.qw), 0, side.cuda_stream)
            if s:
                raise F.Fp8Error(s, "fp8_quantize_ex (weight)")
            L.w_ready.record(side)
        for L in lins:
            stream.wait_event(L.w_ready)
            s = fwd(ctypes.byref(L.fwd_w8), h)
            if s:
                raise F.Fp8Error(s, "fp8_linear_forward")
    stream_handle = h
    for L in reversed(lins):
        s = bwd(ctypes.byref(L.bwd), stream_handle)
        if s:
            raise F.Fp8Error(s, "fp8_linear_backward")


# quantize x+w, fwd GEMM, quantize g (+ dbias partials), dX+dW GEMMs (the
# reported count comes from the captured graph)
LAUNCHES_PER_LINEAR = 4


# --------------------------------------------------------------------------- kernel-level timing

def step_primitives(F, lins, h, split_w=False):
    """The step's kernel launches as (class, algorithmic work, label, call) in
    launch order, through the standalone entry points that do the same work as
    the fused fp8_linear_forward / fp8_linear_backward: quantize x+w, forward
    GEMM (+bias); then in reverse, quantize g (+ dbias), dX+dW GEMMs."""
    lib = F._lib
    out = []
    keep = []  # ctypes argument structs must outlive the calls and the graphs

    def call(fn, *structs):
        keep.append(structs)
        return lambda: fn(*[ctypes.byref(s_) for s_ in structs], h)
    for L in lins:
        M, K, N = L.shape.M, L.shape.K, L.shape.N
        ldk = L.x8.shape[1]
        sc = L.sc.data_ptr()
        qx = F.QuantizeArgs(L.x.data_ptr(), 0, M, K, K, 0, L.rings[0].data_ptr(), wl.HIST_LEN, L.x8.data_ptr(), ldk,
                            sc + 12, sc)
        qw = F.QuantizeArgs(L.w.data_ptr(), 0, N, K, K, 0, L.rings[1].data_ptr(), wl.HIST_LEN, L.w8.data_ptr(), ldk,
                            sc + 16, sc + 4)
        fwd = F.MmArgs(M, N, K, L.x8.data_ptr(), 0, 0, ldk, L.w8.data_ptr(), 0, 0, ldk, sc, sc + 4,
                       L.bias_ptr, L.bias_dtype, L.bias_scale_ptr, L.y.data_ptr(), N, 0)
        if split_w:  # the weight in its own launch (the side-stream schedule), then x
            out.append(("quantize", N * K * 3, None, (lambda qw=qw: lib.fp8_quantize_ex(ctypes.byref(qw), 0, h))))
            out.append(("quantize", M * K * 3, None, (lambda qx=qx: lib.fp8_quantize_ex(ctypes.byref(qx), 0, h))))
            keep.append((qx, qw))
        else:
            out.append(("quantize", (M * K + N * K) * 3, None, call(lib.fp8_quantize_dual, qx, qw)))
        out.append(("gemm", 2 * M * N * K, f"fwd {M}x{N}x{K}", call(lib.fp8_mm, fwd)))
    for L in reversed(lins):
        M, K, N = L.shape.M, L.shape.K, L.shape.N
        ldk, ldn = L.x8.shape[1], L.g8.shape[1]
        sc = L.sc.data_ptr()
        qg = F.QuantizeArgs(L.g.data_ptr(), 0, M, N, N, 1, L.rings[2].data_ptr(), wl.HIST_LEN, L.g8.data_ptr(), ldn,
                            sc + 20, sc + 8)
        dx = F.MmArgs(M, K, N, L.g8.data_ptr(), 1, 0, ldn, L.w8.data_ptr(), 0, 1, ldk, sc + 8, sc + 4,
                      None, 0, None, L.dx.data_ptr(), K, 0)
        dw = F.MmArgs(N, K, M, L.g8.data_ptr(), 1, 1, ldn, L.x8.data_ptr(), 0, 1, ldk, sc + 8, sc,
                      None, 0, None, L.dw.data_ptr(), K, 0)
        if L.db is not None:
            ws = L.ws
            out.append(("quantize", M * N * 3, None,
                        (lambda qg=qg, L=L, ws=ws: lib.fp8_quantize_dbias(ctypes.byref(qg), L.db.data_ptr(),
                                                                          ws.data_ptr(), ws.numel(), h))))
            keep.append((qg,))
        else:
            out.append(("quantize", M * N * 3, None, (lambda qg=qg: lib.fp8_quantize_ex(ctypes.byref(qg), 0, h))))
            keep.append((qg,))
        out.append(("gemm", 4 * M * N * K, f"dX+dW {M}x{N}x{K}", call(lib.fp8_mm_pair, dx, dw)))
    return out, keep


def time_kernels(F, lins, stream, reps=5, split_w=False):
    """Device time of each kernel class of the step: the class's launches (in
    step order, same buffers) captured as one CUDA graph and replayed between
    CUDA events on the launching stream, so host launch gaps are excluded.
    Returns (ms per step by class, work by class, launches by class, per-shape
    GEMM times)."""
    h = stream.cuda_stream
    prims, keep = step_primitives(F, lins, h, split_w)
    res_ms, work, count = {}, {}, {}
    for cls in ("gemm", "quantize"):
        calls = [c for c in prims if c[0] == cls]
        work[cls] = sum(c[1] for c in calls)
        count[cls] = len(calls)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _, _, _, fn in calls:
                st = fn()
                if st:
                    raise F.Fp8Error(st, cls)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        runs = []
        for _ in range(3):  # median of three timed runs of `reps` replays
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            torch.cuda.synchronize()
            runs.append(e0.elapsed_time(e1) / reps)
        res_ms[cls] = statistics.median(runs)
        del g
    # per-shape GEMM times: one graph per distinct GEMM launch of the step, 12 launches each
    shapes = {}
    seen = {}
    for c in prims:
        if c[0] == "gemm":
            seen.setdefault(c[2], c)
    for name, c in seen.items():
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(12):
                c[3]()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / 12
        shapes[name] = {"us": us, "tflops": c[1] / us / 1e6, "note": "same operands back to back (warm L2)"}
        del g
    del keep
    return res_ms, work, count, shapes


# --------------------------------------------------------------------------- target shapes, per operation

def _graph_us(stream, fns, reps=3):
    """Device time of one call of `fns` (cycled) inside a CUDA graph of
    len(fns) * 4 calls: `reps` replays between CUDA events, the median of three
    such runs."""
    g = torch.cuda.CUDAGraph()
    n = len(fns) * 4
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            fns[i % len(fns)]()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    runs = []
    for _ in range(3):
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        runs.append(e0.elapsed_time(e1) * 1e3 / (reps * n))
    del g
    return statistics.median(runs)


def _sets_for(bytes_per_set, floor=320 << 20, cap=12):
    """Operand sets to cycle through so that one pass touches more than L2."""
    return max(2, min(cap, -(-floor // max(1, bytes_per_set))))


def fp8_codes_like_normal(shape, dtype, device):
    """fp8 codes of a N(0, 1) tensor scaled so that 5 sigma maps to the
    format's largest value (what a delayed-scaling quantize of a normal tensor
    produces), as uint8."""
    fmax = 448.0 if dtype == torch.float8_e4m3fn else 57344.0
    v = torch.randn(shape, device=device) * (fmax / 5.0)
    return v.clamp(-fmax, fmax).to(dtype).view(torch.uint8)


def gemm_min_bytes(op: str, M: int, N: int, K: int, bias_bytes: int = 0) -> int:
    """Compulsory DRAM bytes of one GEMM: fp8 operands read once, bf16 output
    written once (fwd MK + NK + 2MN, dX MN + NK + 2MK, dW MN + MK + 2NK)."""
    if op == "fwd":
        return M * K + N * K + 2 * M * N + bias_bytes
    if op == "dX":
        return M * N + N * K + 2 * M * K
    return M * N + M * K + 2 * N * K


def roofline_tflops(flops: float, nbytes: float, peak_tflops: float, hbm_gbs: float) -> float:
    """min(peak, AI x BW) in TFLOP/s for arithmetic intensity AI = flops / bytes."""
    return min(peak_tflops, flops / nbytes * hbm_gbs * 1e9 / 1e12)


def time_target_shapes(F, device, stream, fp8_peak, hbm_gbs):
    """fwd, dX and dW as separate launches (fp8_mm, the layouts the fused
    backward uses) at the production (config 3, the forward with its E4M3
    bias and bias scale) and large (config 4) shapes, each timed warm (the
    same operands back to back: L2 holds what fits) and cold (operand sets
    cycled so that each pass streams more than L2); and the standalone
    quantize of the large activations (cold).  Each GEMM record carries its
    fraction of the measured fp8 peak, of the 4.5 PFLOP/s nominal peak and of
    its own roofline min(peak, AI x HBM bandwidth) -- the HBM term binds only
    the cold case; warm operands come from L2."""
    h = stream.cuda_stream
    sc = torch.ones(3, dtype=torch.float32, device=device)
    sc[2] = 448.0 / 0.04
    gemm = []
    for cfg_id, shapes in ((3, wl.C3_SHAPES), (4, wl.C4_SHAPES)):
        for s in shapes:
            M, K, N = s.M, s.K, s.N
            per_set = M * K + N * K + M * N + 2 * (M * N + M * K + N * K)
            nsets = _sets_for(per_set)
            sets = []
            for i in range(nsets):
                # the codes a delayed-scaling quantize gives normal tensors (amax ~ 5 sigma -> fp8 max):
                # E4M3 x8 / w8 / bias, E5M2 g8 (the tensor core's speed depends a little on the data)
                x8 = fp8_codes_like_normal((M, K), torch.float8_e4m3fn, device)
                w8 = fp8_codes_like_normal((N, K), torch.float8_e4m3fn, device)
                g8 = fp8_codes_like_normal((M, N), torch.float8_e5m2, device)
                b8 = fp8_codes_like_normal((N,), torch.float8_e4m3fn, device)
                y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
                dx = torch.empty((M, K), dtype=torch.bfloat16, device=device)
                dw = torch.empty((N, K), dtype=torch.bfloat16, device=device)
                sets.append((x8, w8, g8, y, dx, dw, b8))
            sp = sc.data_ptr()
            with_bias = cfg_id == 3
            wp, wn = None, 0
            ops = {
                "fwd": lambda t: F.MmArgs(M, N, K, t[0].data_ptr(), 0, 0, K, t[1].data_ptr(), 0, 0, K, sp, sp + 4,
                                          t[6].data_ptr() if with_bias else None, F.FP8_DT_E4M3,
                                          sp + 8 if with_bias else None, t[3].data_ptr(), N, 0, wp, wn),
                "dX": lambda t: F.MmArgs(M, K, N, t[2].data_ptr(), 1, 0, N, t[1].data_ptr(), 0, 1, K, sp, sp + 4,
                                         None, 0, None, t[4].data_ptr(), K, 0, wp, wn),
                "dW": lambda t: F.MmArgs(N, K, M, t[2].data_ptr(), 1, 1, N, t[0].data_ptr(), 0, 1, K, sp, sp + 4,
                                         None, 0, None, t[5].data_ptr(), K, 0, wp, wn),
            }
            flops = 2.0 * M * N * K
            for op, mk in ops.items():
                nbytes = gemm_min_bytes(op, M, N, K, N if (op == "fwd" and with_bias) else 0)
                roof = roofline_tflops(flops, nbytes, fp8_peak, hbm_gbs)
                rec = {"config": cfg_id, "shape": f"M={M} K={K} N={N}", "op": op,
                       "bias": "e4m3 + bias_scale" if (op == "fwd" and with_bias) else None,
                       "gflop": round(flops / 1e9, 2), "min_bytes": nbytes,
                       "ai_flop_per_byte": round(flops / nbytes, 1),
                       "roofline_cold_tflops": round(roof, 1)}
                for mode, ss in (("warm", sets[:1]), ("cold", sets)):
                    args = [mk(t) for t in ss]
                    fns = [(lambda a=a: F._lib.fp8_mm(ctypes.byref(a), h)) for a in args]
                    us = _graph_us(stream, fns)
                    tf = flops / us / 1e6
                    plan = F.fp8_mm_plan(args[0], None, torch.cuda.get_device_properties(device).multi_processor_count)
                    rec["plan"] = {"tile_cfg": plan.tile_cfg, "stream_k_ctas": plan.stream_k_ctas,
                                   "dp_tiles": plan.dp_tiles}
                    rec[mode] = {"us": round(us, 2), "tflops": round(tf, 1),
                                 "frac_measured_peak": round(tf / fp8_peak, 3),
                                 "frac_nominal_4.5PF": round(tf / NOMINAL_FP8_TFLOPS, 3),
                                 "frac_roofline": round(tf / (fp8_peak if mode == "warm" else roof), 3)}
                gemm.append(rec)
            del sets
    quant = []
    # this box's device-to-device copy rate (read + write bytes), for context:
    # the fractions above and below use the measured peak of the pool
    src = torch.ones(1 << 28, dtype=torch.float32, device=device)
    dst = torch.empty_like(src)
    copy_us = _graph_us(stream, [lambda: torch.mul(src, 1.0, out=dst)], reps=5)
    box_copy_gbs = round(2 * 4 * src.numel() / copy_us / 1e3, 1)
    del src, dst
    ring = torch.empty(F.fp8_ring_bytes(wl.HIST_LEN) // 4, dtype=torch.float32, device=device)
    F.fp8_ring_init(ring, wl.HIST_LEN)
    for rows, cols in ((4096, 4096), (4096, 11008), (2048, 6912)):
        per_set = rows * cols * 3
        nsets = _sets_for(per_set)
        sets = [(torch.randn(rows, cols, device=device).to(torch.bfloat16),
                 torch.empty(rows, cols, dtype=torch.uint8, device=device)) for _ in range(nsets)]
        fns = [(lambda x=x, o=o: F._lib.fp8_quantize(x.data_ptr(), 0, rows, cols, cols, 0, ring.data_ptr(),
                                                     wl.HIST_LEN, o.data_ptr(), cols, None, None, h))
               for x, o in sets]
        us = _graph_us(stream, fns)
        gbs = per_set / us / 1e3
        # as the fused linears launch it: the ring step deferred to the GEMM that follows
        qargs = [F.QuantizeArgs(x.data_ptr(), 0, rows, cols, cols, 0, ring.data_ptr(), wl.HIST_LEN, o.data_ptr(),
                                cols, None, None) for x, o in sets]
        dfns = [(lambda a=a: F._lib.fp8_quantize_ex(ctypes.byref(a), F.FP8_QUANTIZE_DEFER_RING_STEP, h))
                for a in qargs]
        dus = _graph_us(stream, dfns)
        F.fp8_ring_finalize(ring, wl.HIST_LEN, F.FP8_E4M3)
        dgbs = per_set / dus / 1e3
        # current (dynamic) scaling: an amax pass, then the cast with fp8_max / amax
        # (algorithmic bytes as above; the amax pass reads the input a second time)
        am = torch.zeros(1, dtype=torch.float32, device=device)
        yfns = [(lambda x=x, o=o: F._lib.fp8_quantize(x.data_ptr(), 0, rows, cols, cols, 0, None, 0, o.data_ptr(),
                                                      cols, am.data_ptr(), None, h)) for x, o in sets]
        yus = _graph_us(stream, yfns)
        ygbs = per_set / yus / 1e3
        quant.append({"shape": f"{rows}x{cols} bf16->e4m3", "us": round(us, 2), "gbs": round(gbs, 1),
                      "frac_hbm": round(gbs / hbm_gbs, 3),
                      "ring_step_deferred": {"us": round(dus, 2), "gbs": round(dgbs, 1),
                                             "frac_hbm": round(dgbs / hbm_gbs, 3)},
                      "current_scaling": {"us": round(yus, 2), "gbs": round(ygbs, 1),
                                          "frac_hbm": round(ygbs / hbm_gbs, 3),
                                          "min_bytes_with_second_read": per_set + rows * cols * 2}})
        del sets, qargs
    # the bias gradient: the backward's fused g quantize + column sums
    # (fp8_quantize_dbias, E5M2, ring finalize and sums in the launch) and the
    # standalone column sum of a bf16 g (fp8_dbias), cold
    dbias = []
    for rows, cols in ((4096, 11008), (2048, 6912), (2048, 4096)):
        nsets = _sets_for(rows * cols * 3)
        gs = [torch.randn(rows, cols, device=device).mul_(1e-3).to(torch.bfloat16) for _ in range(nsets)]
        outs = [torch.empty(rows, cols, dtype=torch.uint8, device=device) for _ in range(nsets)]
        db = torch.empty(cols, dtype=torch.bfloat16, device=device)
        ws = torch.zeros(max(16, F.fp8_dbias_workspace_bytes(rows, cols)), dtype=torch.uint8, device=device)
        qargs = [F.QuantizeArgs(g.data_ptr(), 0, rows, cols, cols, F.FP8_E5M2, ring.data_ptr(), wl.HIST_LEN,
                                o.data_ptr(), cols, None, None) for g, o in zip(gs, outs)]
        qfns = [(lambda a=a: F._lib.fp8_quantize_dbias(ctypes.byref(a), db.data_ptr(), ws.data_ptr(), ws.numel(), h))
                for a in qargs]
        qus = _graph_us(stream, qfns)
        dfns = [(lambda g=g: F._lib.fp8_dbias(g.data_ptr(), 0, rows, cols, cols, None, db.data_ptr(), ws.data_ptr(),
                                               ws.numel(), h)) for g in gs]
        dus = _graph_us(stream, dfns)
        q_gbs, d_gbs = rows * cols * 3 / qus / 1e3, rows * cols * 2 / dus / 1e3
        dbias.append({"shape": f"{rows}x{cols} bf16",
                      "quantize_dbias": {"us": round(qus, 2), "gbs": round(q_gbs, 1),
                                         "frac_hbm": round(q_gbs / hbm_gbs, 3), "bytes_per_elem": 3},
                      "dbias_only": {"us": round(dus, 2), "gbs": round(d_gbs, 1),
                                     "frac_hbm": round(d_gbs / hbm_gbs, 3), "bytes_per_elem": 2}})
        del gs, outs, qargs
    return gemm, quant, box_copy_gbs, dbias


# --------------------------------------------------------------------------- GEMM traffic (ncu summary)

def gemm_source_sha():
    src = os.path.join(ROOT, "fp8_delayed_scaling_03_b200", "csrc", "gemm.cu")
    with open(src, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


TRAFFIC_SUMMARY = {"c4": "gemm_dram_traffic_c4_step.txt", "dim1024": "gemm_dram_traffic_dim1024_layer.txt"}


def gemm_traffic_per_launch(workload=HEADLINE):
    """DRAM bytes per GEMM launch of the workload's step from the committed ncu
    summary, or None when the summary is missing or was taken on a different
    gemm.cu."""
    name = TRAFFIC_SUMMARY.get(workload)
    if name is None:
        return None
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as fh:
        for line in fh:
            if "=" in line and not line.startswith("#"):
                k, v = line.strip().split("=", 1)
                kv[k.strip()] = v.strip()
    if kv.get("gemm_cu_sha256_16") != gemm_source_sha():
        return None
    try:
        return float(kv["dram_bytes_per_gemm_launch"])
    except (KeyError, ValueError):
        return None


# --------------------------------------------------------------------------- CPU oracle

def oracle_sample(tokens: int, seed: int = 1234):
    """The oracle's forward + backward of the headline linears (the three
    M=4096 shapes) on `tokens` tokens: quantize x (with outliers), w and g
    with rings, fwd/dX/dW GEMMs with fp32 accumulation.  The weights are
    quantized whole, as in a training step.  Returns (seconds, flops)."""
    import numpy as np

    import oracle
    flops = 0
    prepared = []
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)  # noqa: E731
    for j, s in enumerate(wl.C4_SHAPES):
        x = wl.normal_with_outliers((tokens, s.K), 1.0, seed + 10 * j, seed + 10 * j + 4)
        w = wl.normal((s.N, s.K), wl.weight_std(s.K), seed + 10 * j + 1)
        g = wl.normal((tokens, s.N), 1e-3, seed + 10 * j + 3)
        prepared.append((s, bits(x), bits(w), bits(g)))
        flops += 6 * tokens * s.N * s.K
    t0 = time.perf_counter()
    for s, x, w, g in prepared:
        rx, rw, rg = oracle.Ring(wl.HIST_LEN), oracle.Ring(wl.HIST_LEN), oracle.Ring(wl.HIST_LEN)
        f = oracle.linear_forward(tokens, s.N, s.K, x, oracle.DT_BF16, w, oracle.DT_BF16, rx, rw, sumabs=False)
        oracle.linear_backward(tokens, s.N, s.K, g, oracle.DT_BF16, rg, f["x8"], oracle.E4M3, f["sx"], f["w8"],
                               oracle.E4M3, f["sw"], sumabs=False)
    return time.perf_counter() - t0, flops


def sample_text(tokens: int) -> str:
    return (f"{tokens} of 4096 tokens of the three M=4096 linears (quantize x/w/g with rings -- the weights "
            f"whole --, fwd+dX+dW GEMMs with fp32 accumulation)")


def oracle_threads():
    import oracle
    return oracle.num_threads()


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_sample(REF_TOKENS)
    secs, flops = [], 0
    for i in range(args.steps):
        s, flops = oracle_sample(REF_TOKENS, seed=4321 + i)
        secs.append(s)
    total = sum(secs)
    value = flops * len(secs) / total / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp8 e4m3/e5m2 (fp32 accumulate)",
            "data": "synthetic", "config": config_dict(HEADLINE),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                             "sample": sample_text(REF_TOKENS) + " per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_dict(workload=HEADLINE, lins=None):
    d = {"workload": WORKLOADS[workload][0], "hist_len": wl.HIST_LEN,
         "timing": "CUDA graph of the step's C-ABI calls, CUDA events, max over ranks"}
    if workload == "c4":
        d.update(M=4096, linears_per_step=3,
                 l2="inputs larger than L2 (step working set ~1.6 GB, 126 MB L2)")
    elif workload == "dim1024":
        d.update(M=2048, layers=wl.BENCH_LAYERS, linears_per_step=wl.BENCH_LAYERS * len(wl.BENCH_LAYER),
                 l2="inputs larger than L2 (step working set ~3 GB, 126 MB L2)")
    else:
        d.update(M=[512, 2048], linears_per_step=len(wl.C3_SHAPES),
                 l2="inputs larger than L2 (step working set ~0.5 GB, 126 MB L2)")
    return d


# --------------------------------------------------------------------------- end to end

def time_e2e(F, lins, host_in, host_out, comp, device, steps):
    """Device time (ms) of `steps` end-to-end steps through the C ABI with host
    buffers: every step copies each linear's inputs (x, w, b, g) in from
    pinned host memory on one stream, runs fp8_linear_forward over the linears
    and fp8_linear_backward in reverse on the compute stream, and copies each
    linear's y, dX, dW, dbias out to pinned host memory on a third stream.
    Events order each linear's kernels after its inputs arrived, each output
    copy after the kernel that wrote it, a step's input copies after the
    previous step's kernels (which read those buffers) and a step's kernels
    after the previous step's output copies (which read what they overwrite).
    The two copy directions run at once on the full-duplex link."""
    h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    fwd, bwd = F._lib.fp8_linear_forward, F._lib.fp8_linear_backward
    ch = comp.cuda_stream
    n = len(lins)
    state = {"comp_done": None, "d2h_done": None}

    def one_step():
        arrived = []
        with torch.cuda.stream(h2d_s):
            if state["comp_done"] is not None:
                h2d_s.wait_event(state["comp_done"])
            for L, hs in zip(lins, host_in):
                for d, h in zip(L.inputs(), hs):
                    d.copy_(h, non_blocking=True)
                e = torch.cuda.Event()
                e.record(h2d_s)
                arrived.append(e)
        y_ready, grads_ready = [None] * n, [None] * n
        with torch.cuda.stream(comp):
            if state["d2h_done"] is not None:
                comp.wait_event(state["d2h_done"])
            for i, L in enumerate(lins):
                comp.wait_event(arrived[i])
                st = fwd(ctypes.byref(L.fwd), ch)
                if st:
                    raise F.Fp8Error(st, "fp8_linear_forward")
                y_ready[i] = torch.cuda.Event()
                y_ready[i].record(comp)
            for i in reversed(range(n)):
                st = bwd(ctypes.byref(lins[i].bwd), ch)
                if st:
                    raise F.Fp8Error(st, "fp8_linear_backward")
                grads_ready[i] = torch.cuda.Event()
                grads_ready[i].record(comp)
            comp_done = torch.cuda.Event()
            comp_done.record(comp)
        with torch.cuda.stream(d2h_s):
            for i, L in enumerate(lins):
                d2h_s.wait_event(y_ready[i])
                host_out[i][0].copy_(L.y, non_blocking=True)
            for i in reversed(range(n)):
                d2h_s.wait_event(grads_ready[i])
                for d, h in zip(lins[i].outputs()[1:], host_out[i][1:]):
                    h.copy_(d, non_blocking=True)
            d2h_done = torch.cuda.Event()
            d2h_done.record(d2h_s)
        state["comp_done"], state["d2h_done"] = comp_done, d2h_done

    one_step()  # warm-up
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    state["comp_done"], state["d2h_done"] = e0, e0
    for _ in range(steps):
        one_step()
    comp.wait_event(state["d2h_done"])
    e1.record(comp)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


# --------------------------------------------------------------------------- main

def working_set_bytes(lins) -> int:
    ts = []
    for L in lins:
        ts += L.inputs() + L.outputs() + [L.x8, L.w8, L.g8]
    return sum(t.numel() * t.element_size() for t in ts)


def graph_kernel_nodes(graph):
    """Kernel nodes of a captured CUDA graph -- the kernel launches one replay
    runs (None when the graph cannot be inspected)."""
    try:
        from cuda.bindings import runtime as rt
        g = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(g, numNodes=0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(g, numNodes=n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        count = 0
        for nd in nodes[:n]:
            err, t = rt.cudaGraphNodeGetType(nd)
            if err == rt.cudaError_t.cudaSuccess and t == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel:
                count += 1
        return count
    except Exception:
        return None


def capture_step(F, lins, stream, warmup, side=None):
    """Eager step (first-launch set-up outside the capture), then the step
    captured as one CUDA graph (kept, so its kernel nodes can be counted) and
    replayed `warmup` times."""
    with torch.cuda.stream(stream):
        run_step(F, lins, stream, side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(graph, stream=stream):
        run_step(F, lins, stream, side)
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    return graph


def time_graph_ms(graph, stream, reps):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def fp8_peak_for(pk, clocks):
    """The measured fp8 denominator: measured bf16 GEMM x the nominal fp8:bf16
    ratio -- the burst figure while the timed region held the maximum SM
    clock with no power-cap reason, the sustained figure (seconds-long loop
    under the power cap) otherwise."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = "sw_power_cap" in clocks.get("reasons", []) or (mhz is not None and mx and mhz < 0.97 * mx)
    key = "bf16_tflops_sustained" if capped and "bf16_tflops_sustained" in pk else "bf16_tflops"
    return pk[key] * FP8_PER_BF16, key


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS),
                    help="workload of the timed step (the headline by default)")
    ap.add_argument("--layers", type=int, default=wl.BENCH_LAYERS, help="layers of the dim1024 workload "
                    "(profiling runs only)")
    ap.add_argument("--no-extras", action="store_true", help="skip e2e, kernel timing, targets and cpu baseline")
    ap.add_argument("--weights", default="fused", choices=["side", "fused"],
                    help="side: weights quantized on a second stream ahead of the forward linears (pre-quantized "
                         "weights), overlapping the earlier GEMMs; fused: x and w quantized in each linear's "
                         "fp8_linear_forward")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    wl.BENCH_LAYERS = args.layers
    if args.impl == "reference":
        return run_reference(args)

    import fp8_delayed_scaling_03_b200 as F

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    lins = build_model(F, device, rank, args.workload)
    stream = torch.cuda.Stream(device)
    side = torch.cuda.Stream(device) if args.weights == "side" else None
    torch.cuda.synchronize()
    flops_step = step_flops(lins)
    graph = capture_step(F, lins, stream, args.warmup, side)

    # ---- timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = time_graph_ms(graph, stream, args.steps)
    if world > 1:
        dist.barrier()
    max_ms = reduce_max(ms, world, device)
    value = aggregate_throughput(flops_step * args.steps, world, max_ms / 1e3) / 1e12
    status = F.fp8_get_device_status()
    if status:
        raise F.Fp8Error(status, "device status after timed region")
    clocks = clk.report()
    cfg = config_dict(args.workload)
    cfg["working_set_bytes"] = working_set_bytes(lins)
    cfg["weights"] = ("quantized on a second stream ahead of the forward linears, which take them pre-quantized "
                      "(each waits for its own weight only)" if side is not None else
                      "quantized with x inside each fp8_linear_forward")

    kernels_per_step = graph_kernel_nodes(graph)
    cfg["kernels_per_step"] = kernels_per_step if kernels_per_step is not None else \
        f"not inspectable; at least {LAUNCHES_PER_LINEAR * len(lins)}"
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8 e4m3/e5m2 (fp32 accumulate, bf16 out)", "data": "synthetic",
            "config": cfg, "clocks": clocks,
            "gpu_launches": (kernels_per_step or LAUNCHES_PER_LINEAR * len(lins)) * args.steps}

    if not args.no_extras:
        pk, pk_kind = peaks()
        fp8_peak, peak_key = fp8_peak_for(pk, clocks)
        # ---- kernel-level timing and roofline of the dominant kernel (the GEMM class)
        tot, work, count, shapes = time_kernels(F, lins, stream, split_w=side is not None)
        gemm_tflops = work["gemm"] / (tot["gemm"] / 1e3) / 1e12
        traffic = gemm_traffic_per_launch(args.workload)
        line["roofline"] = {"bound": "tensor", "achieved": gemm_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                            "frac": gemm_tflops / fp8_peak, "traffic": traffic,
                            "kernel": f"fp8_gemm_kernel (the step's {count['gemm']} GEMM launches: forward and "
                                      f"dX+dW pairs, replayed as one graph)",
                            "peak_source": f"{pk_kind} {peak_key} x {FP8_PER_BF16} (nominal fp8:bf16)",
                            "frac_of_nominal_4.5PF": gemm_tflops / NOMINAL_FP8_TFLOPS}
        # The quantize class is timed as its own graph of the step's quantize
        # calls (each finalizing its ring in its last block).  Inside the
        # fused linears the quantize launches overlap the neighbouring GEMMs'
        # tails (programmatic dependent launch), so "step minus the GEMM
        # class" is the step time the GEMMs do not cover, not a bandwidth.
        step_ms = max_ms / args.steps
        q_gbs = work["quantize"] / (tot["quantize"] / 1e3) / 1e9
        classes = {"gemm": tot["gemm"], "quantize": tot["quantize"]}
        line["kernels"] = {
            "share_of_class_sum": {k: v / sum(classes.values()) for k, v in classes.items()},
            "ms_per_step": classes, "launches_per_step": count,
            "step_minus_gemm_class_ms": max(step_ms - tot["gemm"], 0.0),
            "quantize": {"achieved_gbs": q_gbs, "peak_gbs": pk["hbm_gbs"], "frac": q_gbs / pk["hbm_gbs"],
                         "bytes_per_elem": 3,
                         "note": "bf16 in + fp8 out; x and w in one launch (fused weights) or in two (weights on "
                                 "the side stream), g (with its bias-gradient partials when the bias needs a "
                                 "gradient) in one launch; standalone class graph, each launch finalizing its ring"},
            "gemm_by_shape": shapes}

        # ---- the other workloads' steps, timed the same way
        others = {}
        for wname in WORKLOADS:
            if wname == args.workload:
                continue
            olins = build_model(F, device, rank, wname)
            og = capture_step(F, olins, stream, args.warmup, side)
            oreps = max(5, args.steps // 2)
            if world > 1:
                dist.barrier()
            oms = reduce_max(time_graph_ms(og, stream, oreps), world, device)
            ofl = step_flops(olins)
            ot, owork, ocount, _ = time_kernels(F, olins, stream, split_w=side is not None)
            otf = owork["gemm"] / (ot["gemm"] / 1e3) / 1e12
            others[wname] = {"workload": WORKLOADS[wname][0],
                             "value": aggregate_throughput(ofl * oreps, world, oms / 1e3) / 1e12, "unit": UNIT,
                             "ms_per_step": oms / oreps,
                             "gpu_launches_per_step": graph_kernel_nodes(og) or LAUNCHES_PER_LINEAR * len(olins),
                             "gemm_class": {"tflops": otf, "frac_measured_peak": otf / fp8_peak,
                                            "ms_per_step": ot["gemm"]}}
            del og, olins
            torch.cuda.synchronize()
        if F.fp8_get_device_status():
            raise F.Fp8Error(F.fp8_get_device_status(), "device status after the other workloads")
        line["steps_other_workloads"] = others

        # the per-operation launches run right after the steps above: their
        # SM clock (and any power-cap reason) is sampled and reported with them
        with ClockSampler(local) as tclk:
            tg, tq, box_copy, tdb = time_target_shapes(F, device, stream, fp8_peak, pk["hbm_gbs"])
        line["targets"] = {
            "gemm": tg, "quantize": tq, "dbias": tdb, "fp8_peak_tflops": fp8_peak, "hbm_gbs": pk["hbm_gbs"],
            "box_copy_gbs": box_copy, "clocks": tclk.report(),
            "note": "separate fp8_mm launches per operation (dX, dW in the fused backward's in-place "
                    "transposed layouts); warm = the same operands back to back, cold = operand sets cycled so "
                    "each pass streams more than L2; frac_roofline = achieved / min(peak, AI x HBM BW) cold, "
                    "achieved / peak warm; quantize standalone (in-kernel ring finalize) and with the ring step "
                    "deferred to the following GEMM (as fp8_linear_forward/backward launch it), cold; "
                    "box_copy_gbs = this box's rate for an elementwise 1 GiB -> 1 GiB fp32 copy kernel (read + write bytes), context "
                    "for the HBM fractions, which use the pool's measured peak"}

        # ---- end to end through the C ABI with host buffers
        host_in = [[t.cpu().pin_memory() for t in L.inputs()] for L in lins]
        host_out = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in L.outputs()] for L in lins]
        h2d = sum(t.numel() * t.element_size() for ts in host_in for t in ts)
        d2h = sum(t.numel() * t.element_size() for ts in host_out for t in ts)

        e2e_steps = max(3, min(args.steps, 10))
        if world > 1:
            dist.barrier()
        e2e_ms = reduce_max(time_e2e(F, lins, host_in, host_out, stream, device, e2e_steps), world, device)
        line["e2e"] = {"value": aggregate_throughput(flops_step * e2e_steps, world, e2e_ms / 1e3) / 1e12,
                       "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": e2e_ms / e2e_steps, "steps": e2e_steps,
                       "path": "pinned host -> device copies of each linear's inputs (copy stream), "
                               "fp8_linear_forward/backward per linear (compute stream), device -> pinned host copies "
                               "of its outputs (second copy stream); per-linear events, so the two copy directions "
                               "and the kernels overlap"}

        # ---- CPU oracle baseline (rank 0, one GPU only)
        if rank == 0 and world == 1:
            secs, flops = oracle_sample(CPU_SAMPLE_TOKENS)
            line["cpu_baseline"] = {"value": flops / secs / 1e12, "unit": UNIT, "cores": oracle_threads(),
                                    "kind": "oracle", "sample": sample_text(CPU_SAMPLE_TOKENS) + f", {secs:.1f} s"}

    if world > 1:
        del graph
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
