"""CPU oracle for the FP8 linear layer with delayed scaling.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by the smoke check and by
the CPU-baseline leg of ``bench.py``; never by the product package, which
shares no code with it.

The arithmetic lives in ``fp8_oracle.c`` (plain C, OpenMP over independent
output rows); this module marshals numpy arrays and holds the orchestration of
the pages' forward/backward step (which operand is quantized with which ring,
which scale each GEMM dequantizes with).  Sources, by page of the AstrAI commit
log:

* scale ring folded inside the quantize kernel, ``[hist | scale | counter]``:
  ``tests/extension @2eeac02``, ring-finalize bullets;
* pre-quantized operands skip their quantize, amax 0:
  ``tests/extension @2eeac02``, w8 bullet; ``astrai/extension/ops @057c0d3``;
* snapshot of sx/sw/sg before the ring overwrites the scale, backward reuses
  the forward's scales, grads in bf16, pre-quantized g dequantized before the
  bias sum: ``astrai/extension/ops @057c0d3``;
* bias fused before the single bf16 rounding, fp8 bias with its own scale:
  ``astrai @4019dda`` fused-bias bullet; ``csrc @2eeac02`` FP8Params bias bullet;
* amax of the raw (not quantized) values: ``astrai/extension/fp8.py @3e57cc8``.

Arrays: bf16 and fp16 tensors are passed as ``np.uint16`` bit patterns, fp32 as
``np.float32``, fp8 as ``np.uint8`` codes.  2-D arrays are row-major; their
second dimension is the row stride (``ld``) and ``cols`` may be smaller.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

E4M3, E5M2 = 0, 1
DT_BF16, DT_FP16, DT_FP32, DT_E4M3, DT_E5M2 = 0, 1, 2, 3, 4
FP8_MAX = {E4M3: 448.0, E5M2: 57344.0}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=gnu11",
          "-Wall", "-Wextra", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile the oracle's C file into ``oracle/_build/liboracle.so``."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I64, I, F, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        L.orc_decode_table.argtypes = [I, P]
        L.orc_fp8_max.argtypes = [I]; L.orc_fp8_max.restype = D
        L.orc_encode.argtypes = [I, F]; L.orc_encode.restype = ctypes.c_uint8
        L.orc_encode_array.argtypes = [I, P, I64, P]
        L.orc_bf16_rne.argtypes = [F]; L.orc_bf16_rne.restype = ctypes.c_uint16
        L.orc_bf16_rne_array.argtypes = [P, I64, P]
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]; L.orc_bf16_to_f32.restype = F
        L.orc_fp16_to_f32.argtypes = [ctypes.c_uint16]; L.orc_fp16_to_f32.restype = F
        L.orc_amax.argtypes = [P, I, I64, I64, I64]; L.orc_amax.restype = F
        L.orc_quantize.argtypes = [P, I, I64, I64, I64, I, F, P, I64]
        L.orc_ring_step.argtypes = [P, I, P, F, F, I]; L.orc_ring_step.restype = F
        L.orc_gemm.argtypes = [I64, I64, I64, P, I, I64, I64, P, I, I64, I64, P, P, P]
        L.orc_gemm_points.argtypes = [I64, P, P, I64, P, I, I64, I64, P, I, I64, I64, P, P]
        L.orc_epilogue.argtypes = [I64, I64, P, F, F, P, I, F, P, P, P]
        L.orc_dbias.argtypes = [P, I, I64, I64, I64, F, P, P, P]
        L.orc_num_threads.restype = I
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().orc_num_threads()


# ------------------------------------------------------------------ formats

def decode_table(fmt: int) -> np.ndarray:
    out = np.empty(256, np.float64)
    lib().orc_decode_table(fmt, _p(out))
    return out


def decode(fmt: int, codes: np.ndarray) -> np.ndarray:
    """fp8 codes -> exact values (float64)."""
    return decode_table(fmt)[codes.astype(np.int64)]


def encode(fmt: int, v) -> np.ndarray:
    """Saturating RNE cast of fp32 values to fp8 codes."""
    v = np.ascontiguousarray(np.asarray(v, np.float32))
    out = np.empty(v.shape, np.uint8)
    lib().orc_encode_array(fmt, _p(v), v.size, _p(out))
    return out


def bf16_rne(v) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even."""
    v = np.ascontiguousarray(np.asarray(v, np.float32))
    out = np.empty(v.shape, np.uint16)
    lib().orc_bf16_rne_array(_p(v), v.size, _p(out))
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def to_f32(x: np.ndarray, dtype: int) -> np.ndarray:
    """Input tensor (bit patterns) -> fp32 values, exactly."""
    if dtype == DT_BF16:
        return bf16_to_f32(x)
    if dtype == DT_FP16:
        return x.view(np.float16).astype(np.float32)
    if dtype == DT_FP32:
        return x.astype(np.float32)
    raise ValueError(dtype)


# ------------------------------------------------------------------ quantize

def amax(x: np.ndarray, dtype: int, cols: int | None = None) -> np.float32:
    x = np.ascontiguousarray(x)
    rows, ld = x.shape
    cols = ld if cols is None else cols
    return np.float32(lib().orc_amax(_p(x), dtype, rows, cols, ld))


def quantize_codes(x: np.ndarray, dtype: int, fmt: int, s: float, cols: int | None = None,
                   ld_out: int | None = None) -> np.ndarray:
    """q = encode(fp32(x) * s) -> uint8 [rows, ld_out]; pad bytes zero."""
    x = np.ascontiguousarray(x)
    rows, ld = x.shape
    cols = ld if cols is None else cols
    ld_out = cols if ld_out is None else ld_out
    out = np.empty((rows, ld_out), np.uint8)
    lib().orc_quantize(_p(x), dtype, rows, cols, ld, fmt, np.float32(s), _p(out), ld_out)
    return out


# ------------------------------------------------------------------ ring

@dataclass
class Ring:
    """Delayed-scaling state of one tensor: amax history, current scale, step."""
    H: int
    hist: np.ndarray = field(default=None)
    scale: np.float32 = np.float32(1.0)
    step: int = 0

    def __post_init__(self):
        if self.hist is None:
            self.hist = np.zeros(self.H, np.float32)

    def copy(self) -> "Ring":
        return Ring(self.H, self.hist.copy(), np.float32(self.scale), self.step)

    def seed(self, amax_value: float, fmt: int) -> None:
        """Fresh state with scale fp8_max / amax (1.0 unless amax > 0, finite and
        the quotient finite); history zero, step 0."""
        self.hist[:] = 0
        self.step = 0
        a = np.float32(amax_value)
        s = np.float32(1.0)
        if np.isfinite(a) and a > 0:
            with np.errstate(over="ignore"):
                q = np.float32(FP8_MAX[fmt]) / a
            if np.isfinite(q):
                s = np.float32(q)
        self.scale = s

    def advance(self, amax_value: float, fmt: int) -> np.float32:
        step = ctypes.c_uint32(self.step)
        self.scale = np.float32(lib().orc_ring_step(_p(self.hist), self.H, ctypes.byref(step),
                                                    np.float32(self.scale), np.float32(amax_value), fmt))
        self.step = step.value
        return self.scale


def dynamic_scale(amax_value: float, fmt: int) -> np.float32:
    """Current (dynamic) scaling, the pages' alternative to the ring (AstrAI
    commits: astrai @4019dda, recipe bullet -- one recipe with a dynamic flag;
    astrai/extension/fp8.py @3e57cc8, DynamicScaling bullet -- no rings, the
    scale measured inline): the scale of a tensor is fp8_max / its own amax,
    one fp32 IEEE division, and 1.0 when amax is 0, not finite, or the
    quotient overflows (the ring's keep rule with 1.0 as the kept scale)."""
    a = np.float32(amax_value)
    if not (np.isfinite(a) and a > 0):
        return np.float32(1.0)
    with np.errstate(over="ignore"):
        q = np.float32(np.float32(FP8_MAX[fmt]) / a)
    return q if np.isfinite(q) else np.float32(1.0)


def quantize_dynamic(x: np.ndarray, dtype: int, fmt: int, cols: int | None = None,
                     ld_out: int | None = None):
    """Quantize with the tensor's own scale: amax over the raw input first, then
    s = dynamic_scale(amax), then the same cast.  Returns (codes, amax, s)."""
    a = amax(x, dtype, cols)
    s = dynamic_scale(a, fmt)
    q = quantize_codes(x, dtype, fmt, s, cols, ld_out)
    return q, a, s


def quantize(x: np.ndarray, dtype: int, fmt: int, ring: Ring, cols: int | None = None,
             ld_out: int | None = None):
    """One quantize launch as the pages define it: read the ring's current scale
    (the snapshot), reduce amax over the raw input, cast, then fold amax into the
    ring.  Returns (codes, amax, scale_used); ``ring`` is advanced in place."""
    s = np.float32(ring.scale)
    a = amax(x, dtype, cols)
    q = quantize_codes(x, dtype, fmt, s, cols, ld_out)
    ring.advance(a, fmt)
    return q, a, s


# ------------------------------------------------------------------ GEMM

def gemm_acc(a: np.ndarray, fmt_a: int, a_si: int, a_sk: int,
             b: np.ndarray, fmt_b: int, b_sj: int, b_sk: int,
             I: int, J: int, Kc: int, exact: bool = False, sumabs: bool = True):
    """sum_k A(i,k) B(j,k) with fp32 accumulation in k order (and optionally the
    exact dot and sum |ab|).  A(i,k) = a.flat[i*a_si + k*a_sk], same for B."""
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    acc = np.empty((I, J), np.float32)
    ex = np.empty((I, J), np.float64) if exact else None
    sa = np.empty((I, J), np.float64) if sumabs else None
    lib().orc_gemm(I, J, Kc, _p(a), fmt_a, a_si, a_sk, _p(b), fmt_b, b_sj, b_sk,
                   _p(acc), _p(ex), _p(sa))
    return acc, ex, sa


def gemm_acc_points(ii, jj, a, fmt_a, a_si, a_sk, b, fmt_b, b_sj, b_sk, Kc):
    ii = np.ascontiguousarray(ii, np.int64)
    jj = np.ascontiguousarray(jj, np.int64)
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    acc = np.empty(ii.shape, np.float32)
    sa = np.empty(ii.shape, np.float64)
    lib().orc_gemm_points(ii.size, _p(ii), _p(jj), Kc, _p(a), fmt_a, a_si, a_sk,
                          _p(b), fmt_b, b_sj, b_sk, _p(acc), _p(sa))
    return acc, sa


def epilogue(acc: np.ndarray, sa: float, sb: float, bias: np.ndarray | None = None,
             bias_dtype: int = DT_BF16, bias_scale: float = 1.0, col_idx: np.ndarray | None = None):
    """acc / (sa*sb) (+ bias) in fp32, one RNE rounding to bf16.  Returns
    (bf16 bits, fp32 pre-rounding values)."""
    acc = np.ascontiguousarray(acc, np.float32)
    shape = acc.shape
    if acc.size == 0:  # an empty output
        return np.zeros(shape, np.uint16), np.zeros(shape, np.float32)
    acc2 = acc.reshape(1, -1) if col_idx is not None else acc.reshape(shape[0] if acc.ndim > 1 else 1, -1)
    out = np.empty(acc2.shape, np.uint16)
    f = np.empty(acc2.shape, np.float32)
    ci = None if col_idx is None else np.ascontiguousarray(col_idx, np.int64).reshape(-1)
    bias_c = None if bias is None else np.ascontiguousarray(bias)
    lib().orc_epilogue(acc2.shape[0], acc2.shape[1], _p(acc2), np.float32(sa), np.float32(sb),
                       _p(bias_c), bias_dtype, np.float32(bias_scale), _p(ci), _p(out), _p(f))
    return out.reshape(shape), f.reshape(shape)


# Operand views of the three GEMMs.  X8 [M,K] (row stride ldx), W8 [N,K] (ldw),
# G8 [M,N] (ldg); the contraction index is the last argument of A(i,k)/B(j,k).

def fwd_acc(x8, ldx, fmt_x, w8, ldw, fmt_w, M, N, K, **kw):
    """Y[m,n] = sum_k X8[m,k] W8[n,k]."""
    return gemm_acc(x8, fmt_x, ldx, 1, w8, fmt_w, ldw, 1, M, N, K, **kw)


def dx_acc(g8, ldg, fmt_g, w8, ldw, fmt_w, M, N, K, **kw):
    """dX[m,k] = sum_n G8[m,n] W8[n,k]."""
    return gemm_acc(g8, fmt_g, ldg, 1, w8, fmt_w, 1, ldw, M, K, N, **kw)


def dw_acc(g8, ldg, fmt_g, x8, ldx, fmt_x, M, N, K, **kw):
    """dW[n,k] = sum_m G8[m,n] X8[m,k]."""
    return gemm_acc(g8, fmt_g, 1, ldg, x8, fmt_x, 1, ldx, N, K, M, **kw)


# ------------------------------------------------------------------ dbias

def dbias(g: np.ndarray, dtype: int, M: int, N: int, sg: float = 1.0):
    """bf16( sum_m g[m,n] ) with fp32 accumulation, m ascending; fp8 g is
    dequantized (decode / sg) before the sum.  Returns (bf16 bits, fp32 sums,
    sum |g| per column)."""
    g = np.ascontiguousarray(g)
    ld = g.shape[1]
    out = np.empty(N, np.uint16)
    f = np.empty(N, np.float32)
    sa = np.empty(N, np.float64)
    lib().orc_dbias(_p(g), dtype, M, N, ld, np.float32(sg), _p(out), _p(f), _p(sa))
    return out, f, sa


# ------------------------------------------------------------------ orchestration

def _operand(t, dtype, fmt, ring, scale_in, cols, ld8):
    """Quantize an operand with its ring, or take a pre-quantized one as is.
    An operand with no elements is not quantized: it has no amax to fold, so
    its ring does not step (the pages are silent on empty tensors; reading: a
    quantize of nothing does nothing) and the scale returned is the one a
    quantize would have used."""
    if dtype in (DT_E4M3, DT_E5M2):
        assert (dtype - DT_E4M3) == fmt, "pre-quantized operand must match fmt"
        return np.ascontiguousarray(t), np.float32(0.0), np.float32(scale_in)
    if t.size == 0 or (cols is not None and cols == 0):
        rows = t.shape[0]
        width = cols if ld8 is None else ld8
        s = np.float32(1.0) if ring is None else np.float32(ring.scale)
        return np.zeros((rows, width if width is not None else t.shape[1]), np.uint8), np.float32(0.0), s
    if ring is None:  # current (dynamic) scaling
        return quantize_dynamic(t, dtype, fmt, cols=cols, ld_out=ld8)
    q, a, s = quantize(t, dtype, fmt, ring, cols=cols, ld_out=ld8)
    return q, a, s


def linear_forward(M, N, K, x, x_dtype, w, w_dtype, ring_x: Ring | None, ring_w: Ring | None,
                   fmt_x=E4M3, fmt_w=E4M3, bias=None, bias_dtype=DT_BF16, bias_scale=1.0,
                   x_scale_in=1.0, w_scale_in=1.0, ldx8=None, ldw8=None, sumabs=True):
    """Forward of the FP8 linear: quantize x and w (each with its own ring,
    with its own amax when the ring is None, or skipped when pre-quantized),
    then Y = bf16(X8 W8^T / (sx sw) + bias).
    Returns a dict with y (bf16 bits), x8, w8, the scale snapshots sx, sw, the
    amaxes, the fp32 accumulator and sum|ab|."""
    x8, ax, sx = _operand(x, x_dtype, fmt_x, ring_x, x_scale_in, K, ldx8)
    w8, aw, sw = _operand(w, w_dtype, fmt_w, ring_w, w_scale_in, K, ldw8)
    acc, _, sab = fwd_acc(x8, x8.shape[1], fmt_x, w8, w8.shape[1], fmt_w, M, N, K, sumabs=sumabs)
    y, yf = epilogue(acc, sx, sw, bias, bias_dtype, bias_scale)
    return dict(y=y, y_f32=yf, x8=x8, w8=w8, sx=sx, sw=sw, amax_x=ax, amax_w=aw, acc=acc, sumabs=sab)


def linear_backward(M, N, K, g, g_dtype, ring_g: Ring | None, x8, fmt_x, sx, w8, fmt_w, sw,
                    fmt_g=E5M2, g_scale_in=1.0, ldg8=None, need_dx=True, need_dw=True,
                    need_dbias=False, sumabs=True):
    """Backward: quantize g with its ring (E5M2; skipped when pre-quantized),
    dX = bf16(G8 W8 / (sg sw)), dW = bf16(G8^T X8 / (sg sx)) using the
    forward's snapshots sx, sw, and dbias = bf16(sum_m g) from the raw g (or
    g8 / sg when g arrived quantized)."""
    g8, ag, sg = _operand(g, g_dtype, fmt_g, ring_g, g_scale_in, N, ldg8)
    out = dict(g8=g8, sg=sg, amax_g=ag)
    if need_dx:
        acc, _, sab = dx_acc(g8, g8.shape[1], fmt_g, w8, w8.shape[1], fmt_w, M, N, K, sumabs=sumabs)
        out["dx"], out["dx_f32"] = epilogue(acc, sg, sw)
        out["dx_acc"], out["dx_sumabs"] = acc, sab
    if need_dw:
        acc, _, sab = dw_acc(g8, g8.shape[1], fmt_g, x8, x8.shape[1], fmt_x, M, N, K, sumabs=sumabs)
        out["dw"], out["dw_f32"] = epilogue(acc, sg, sx)
        out["dw_acc"], out["dw_sumabs"] = acc, sab
    if need_dbias:
        if g_dtype in (DT_E4M3, DT_E5M2):
            out["dbias"], out["dbias_f32"], out["dbias_sumabs"] = dbias(g8, g_dtype, M, N, sg)
        else:
            out["dbias"], out["dbias_f32"], out["dbias_sumabs"] = dbias(g, g_dtype, M, N)
    return out


# ------------------------------------------------------------------ tolerance

def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |v| (v given as fp32/fp64 values); for zero and
    subnormals the smallest subnormal spacing 2^-133."""
    a = np.abs(np.asarray(v, np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, np.ldexp(1.0, (e - 7).astype(np.int64)), np.ldexp(1.0, -133))


def gemm_tolerance(y_oracle_bf16: np.ndarray, sumabs: np.ndarray, sa: float, sb: float) -> np.ndarray:
    """Allowed |y_gpu - y_oracle| per element: max(1 bf16 ulp of the oracle
    value, 2e-6 * sum_k |a_k b_k| / (sa sb))."""
    yo = bf16_to_f32(y_oracle_bf16).astype(np.float64)
    return np.maximum(bf16_ulp(yo), 2e-6 * sumabs / (float(sa) * float(sb)))
