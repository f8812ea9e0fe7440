"""FP8 linear layer with delayed scaling for B200 (sm_100a).

Thin ctypes binding of ``libfp8lin.so`` (declared in ``include/fp8lin.h``).
Every step of the path runs in the library's CUDA kernels; this module only
marshals tensors into pointers, sizes and the current CUDA stream.  PyTorch
supplies device memory and streams.  There is no CPU fallback: importing the
package without the built library raises.

Entry points carry the C names (``fp8_quantize``, ``fp8_mm``, ...).  A few
helpers (``ScaleRing``, ``quantize``, ``linear_forward``, ``linear_backward``)
allocate outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libfp8lin.so")

FP8_E4M3, FP8_E5M2 = 0, 1
FP8_DT_BF16, FP8_DT_FP16, FP8_DT_FP32, FP8_DT_E4M3, FP8_DT_E5M2 = 0, 1, 2, 3, 4
FP8_K_MAJOR, FP8_MN_MAJOR = 0, 1
FP8_TILE_AUTO, FP8_TILE_128x128, FP8_TILE_128x256, FP8_TILE_PAIR_256x256, FP8_TILE_SPLITK_128x128 = 0, 1, 2, 3, 4
FP8_TILE_STREAMK = 8
FP8_OK = 0
FP8_ERR_INVALID_ARG, FP8_ERR_UNSUPPORTED, FP8_ERR_MISALIGNED = -1, -2, -3
FP8_ERR_CUDA, FP8_ERR_DEVICE_TIMEOUT, FP8_ERR_WORKSPACE = -4, -5, -6
FP8_ERR_TOO_LARGE = -7
FP8_MAX = {FP8_E4M3: 448.0, FP8_E5M2: 57344.0}


class Fp8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status} ({fp8_status_string(status)})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python fp8_delayed_scaling_03_b200/build.py` "
                      "(there is no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)
_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class MmArgs(ctypes.Structure):
    _fields_ = [("m", _I64), ("n", _I64), ("k", _I64),
                ("a", _P), ("fmt_a", _I), ("a_major", _I), ("lda", _I64),
                ("b", _P), ("fmt_b", _I), ("b_major", _I), ("ldb", _I64),
                ("scale_a", _P), ("scale_b", _P),
                ("bias", _P), ("bias_dtype", _I), ("bias_scale", _P),
                ("d", _P), ("ldd", _I64),
                ("tile_cfg", _I),
                ("workspace", _P), ("workspace_bytes", _SZ)]


class MmPlanInfo(ctypes.Structure):
    _fields_ = [("tile_cfg", _I), ("tiles", _I64), ("units", _I), ("est_us", ctypes.c_double),
                ("stream_k_ctas", _I), ("dp_tiles", _I64)]


class QuantizeArgs(ctypes.Structure):
    _fields_ = [("in_", _P), ("in_dtype", _I), ("rows", _I64), ("cols", _I64), ("ld_in", _I64),
                ("fmt", _I), ("ring", _P), ("hist_len", _I),
                ("out", _P), ("ld_out", _I64),
                ("amax_out", _P), ("scale_out", _P)]


class LinearFwdArgs(ctypes.Structure):
    _fields_ = [("M", _I64), ("N", _I64), ("K", _I64),
                ("x", _P), ("x_dtype", _I), ("ldx", _I64), ("x_scale_in", _P),
                ("w", _P), ("w_dtype", _I), ("ldw", _I64), ("w_scale_in", _P),
                ("bias", _P), ("bias_dtype", _I), ("bias_scale", _P),
                ("fmt_x", _I), ("fmt_w", _I), ("hist_len", _I),
                ("ring_x", _P), ("ring_w", _P),
                ("x8", _P), ("ldx8", _I64),
                ("w8", _P), ("ldw8", _I64),
                ("sx_out", _P), ("sw_out", _P), ("amax_x_out", _P), ("amax_w_out", _P),
                ("y", _P), ("ldy", _I64)]


class LinearBwdArgs(ctypes.Structure):
    _fields_ = [("M", _I64), ("N", _I64), ("K", _I64),
                ("g", _P), ("g_dtype", _I), ("ldg", _I64), ("g_scale_in", _P),
                ("fmt_g", _I), ("hist_len", _I), ("ring_g", _P),
                ("g8", _P), ("ldg8", _I64),
                ("sg_out", _P), ("amax_g_out", _P),
                ("x8", _P), ("ldx8", _I64), ("sx", _P), ("fmt_x", _I),
                ("w8", _P), ("ldw8", _I64), ("sw", _P), ("fmt_w", _I),
                ("need_dx", _I), ("need_dw", _I), ("need_dbias", _I),
                ("dx", _P), ("lddx", _I64),
                ("dw", _P), ("lddw", _I64),
                ("dbias", _P),
                ("workspace", _P), ("workspace_bytes", _SZ)]


_SIGS = {
    "fp8_ring_bytes": (_SZ, [_I]),
    "fp8_ring_init": (_I, [_P, _I, _P]),
    "fp8_ring_seed": (_I, [_P, _I, _I, _F, _P]),
    "fp8_quantize": (_I, [_P, _I, _I64, _I64, _I64, _I, _P, _I, _P, _I64, _P, _P, _P]),
    "fp8_quantize_dual": (_I, [ctypes.POINTER(QuantizeArgs), ctypes.POINTER(QuantizeArgs), _P]),
    "fp8_quantize_dbias": (_I, [ctypes.POINTER(QuantizeArgs), _P, _P, _SZ, _P]),
    "fp8_mm": (_I, [ctypes.POINTER(MmArgs), _P]),
    "fp8_mm_plan": (_I, [ctypes.POINTER(MmArgs), ctypes.POINTER(MmArgs), _I, ctypes.POINTER(MmPlanInfo)]),
    "fp8_mm_pair": (_I, [ctypes.POINTER(MmArgs), ctypes.POINTER(MmArgs), _P]),
    "fp8_mm_batched": (_I, [ctypes.POINTER(MmArgs), _I64, _I64, _I64, _I64, _P]),
    "fp8_mm_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "fp8_quantize_ex": (_I, [ctypes.POINTER(QuantizeArgs), _I, _P]),
    "fp8_ring_finalize": (_I, [_P, _I, _I, _P, _P]),
    "fp8_dbias_workspace_bytes": (_SZ, [_I64, _I64]),
    "fp8_dbias": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _P, _SZ, _P]),
    "fp8_dbias_noalloc": (_I, [_P, _I, _I64, _I64, _I64, _P, _P, _P]),
    "fp8_linear_forward": (_I, [ctypes.POINTER(LinearFwdArgs), _P]),
    "fp8_linear_backward": (_I, [ctypes.POINTER(LinearBwdArgs), _P]),
    "fp8_linear_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "fp8_get_device_status": (_I, []),
    "fp8_wait_selftest": (_I, [_P, ctypes.c_uint64, _P, _P]),
    "fp8_status_string": (ctypes.c_char_p, [_I]),
    "fp8_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EXPORTED = tuple(_SIGS)

# --------------------------------------------------------------------------- helpers


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(device=None):
    return torch.cuda.current_stream(device).cuda_stream


def _check(status: int, where: str):
    if status != FP8_OK:
        raise Fp8Error(status, where)


def _dtype_code(t: torch.Tensor, fp8_fmt: int | None = None) -> int:
    """torch dtype -> FP8_DT_*; uint8 tensors are fp8 codes of `fp8_fmt`."""
    if t.dtype == torch.bfloat16:
        return FP8_DT_BF16
    if t.dtype == torch.float16:
        return FP8_DT_FP16
    if t.dtype == torch.float32:
        return FP8_DT_FP32
    if t.dtype == torch.float8_e4m3fn:
        return FP8_DT_E4M3
    if t.dtype == torch.float8_e5m2:
        return FP8_DT_E5M2
    if t.dtype == torch.uint8 and fp8_fmt is not None:
        return FP8_DT_E4M3 + fp8_fmt
    raise TypeError(f"unsupported dtype {t.dtype}")


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _ld(t: torch.Tensor) -> int:
    """Row stride (elements) of a 2-D tensor whose last dim is contiguous."""
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with a contiguous last dimension")
    return t.stride(0)


def fp8_alloc(rows: int, cols: int, device) -> torch.Tensor:
    """fp8 code buffer [rows, ld] with ld = cols rounded up to 16 (the TMA rule),
    returned as the [rows, cols] view."""
    ld = (cols + 15) // 16 * 16
    return torch.zeros((rows, ld), dtype=torch.uint8, device=device)[:, :cols]


# --------------------------------------------------------------------------- C names

def fp8_ring_bytes(hist_len: int) -> int:
    return _lib.fp8_ring_bytes(hist_len)


def fp8_ring_init(ring: torch.Tensor, hist_len: int) -> None:
    _check(_lib.fp8_ring_init(_ptr(ring), hist_len, _stream(ring.device)), "fp8_ring_init")


def fp8_ring_seed(ring: torch.Tensor, hist_len: int, fmt: int, amax: float) -> None:
    _check(_lib.fp8_ring_seed(_ptr(ring), hist_len, fmt, amax, _stream(ring.device)), "fp8_ring_seed")


def fp8_quantize(x: torch.Tensor, fmt: int, ring: torch.Tensor, hist_len: int, out: torch.Tensor,
                 amax_out: torch.Tensor | None = None, scale_out: torch.Tensor | None = None) -> None:
    rows, cols = x.shape
    _check(_lib.fp8_quantize(_ptr(x), _dtype_code(x), rows, cols, _ld(x), fmt, _ptr(ring), hist_len,
                             _ptr(out), _ld(out), _ptr(amax_out), _ptr(scale_out), _stream(x.device)),
           "fp8_quantize")


def quantize_args(x: torch.Tensor, fmt: int, ring: torch.Tensor, hist_len: int, out: torch.Tensor,
                  amax_out: torch.Tensor | None = None, scale_out: torch.Tensor | None = None) -> QuantizeArgs:
    rows, cols = x.shape
    return QuantizeArgs(_ptr(x), _dtype_code(x), rows, cols, _ld(x), fmt, _ptr(ring), hist_len, _ptr(out), _ld(out),
                        _ptr(amax_out), _ptr(scale_out))


FP8_QUANTIZE_DEFER_RING_STEP = 1


def fp8_quantize_ex(a: QuantizeArgs, flags: int, device=None) -> None:
    _check(_lib.fp8_quantize_ex(ctypes.byref(a), flags, _stream(device)), "fp8_quantize_ex")


def fp8_ring_finalize(ring: torch.Tensor, hist_len: int, fmt: int, amax_out: torch.Tensor | None = None) -> None:
    _check(_lib.fp8_ring_finalize(_ptr(ring), hist_len, fmt, _ptr(amax_out), _stream(ring.device)),
           "fp8_ring_finalize")


def fp8_quantize_dual(a: QuantizeArgs, b: QuantizeArgs, device=None) -> None:
    _check(_lib.fp8_quantize_dual(ctypes.byref(a), ctypes.byref(b), _stream(device)), "fp8_quantize_dual")


def fp8_quantize_dbias(g: QuantizeArgs, dbias: torch.Tensor, workspace: torch.Tensor) -> None:
    _check(_lib.fp8_quantize_dbias(ctypes.byref(g), _ptr(dbias), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(dbias.device)),
           "fp8_quantize_dbias")


def fp8_mm_pair(a: MmArgs, b: MmArgs, device=None) -> None:
    _check(_lib.fp8_mm_pair(ctypes.byref(a), ctypes.byref(b), _stream(device)), "fp8_mm_pair")


def fp8_mm_batched(a: MmArgs, batch: int, stride_a: int, stride_b: int, stride_d: int, device=None) -> None:
    """batch GEMMs of a's shape; element strides between batches (0 shares an operand)."""
    _check(_lib.fp8_mm_batched(ctypes.byref(a), batch, stride_a, stride_b, stride_d, _stream(device)),
           "fp8_mm_batched")


def fp8_mm(m, n, k, a, fmt_a, a_major, lda, b, fmt_b, b_major, ldb, scale_a, scale_b, d, ldd,
           bias=None, bias_dtype=FP8_DT_BF16, bias_scale=None, stream=None, tile_cfg=FP8_TILE_AUTO,
           workspace=None) -> None:
    args = MmArgs(m, n, k, _ptr(a), fmt_a, a_major, lda, _ptr(b), fmt_b, b_major, ldb,
                  _ptr(scale_a), _ptr(scale_b), _ptr(bias), bias_dtype, _ptr(bias_scale), _ptr(d), ldd, tile_cfg,
                  _ptr(workspace), _nbytes(workspace))
    s = stream if stream is not None else _stream(d.device if isinstance(d, torch.Tensor) else None)
    _check(_lib.fp8_mm(ctypes.byref(args), s), "fp8_mm")


def fp8_mm_workspace_bytes(m: int, n: int, k: int) -> int:
    return _lib.fp8_mm_workspace_bytes(m, n, k)


def mm_workspace(m: int, n: int, k: int, device) -> torch.Tensor | None:
    """A zero-filled stream-K workspace for GEMMs of this size (None when empty)."""
    nb = fp8_mm_workspace_bytes(m, n, k)
    return torch.zeros(nb, dtype=torch.uint8, device=device) if nb else None


def fp8_mm_plan(a: MmArgs, b: MmArgs | None = None, num_sms: int = 148) -> MmPlanInfo:
    """The tile configuration fp8_mm (or fp8_mm_pair with b) would choose on a
    GPU with num_sms SMs; host arithmetic only (no device needed)."""
    info = MmPlanInfo()
    _check(_lib.fp8_mm_plan(ctypes.byref(a), ctypes.byref(b) if b is not None else None, num_sms,
                            ctypes.byref(info)), "fp8_mm_plan")
    return info


def fp8_dbias_workspace_bytes(M: int, N: int) -> int:
    return _lib.fp8_dbias_workspace_bytes(M, N)


def fp8_dbias(g: torch.Tensor, dbias: torch.Tensor, workspace: torch.Tensor,
              g_scale: torch.Tensor | None = None, g_fmt: int | None = None) -> None:
    M, N = g.shape
    _check(_lib.fp8_dbias(_ptr(g), _dtype_code(g, g_fmt), M, N, _ld(g), _ptr(g_scale), _ptr(dbias),
                          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(g.device)),
           "fp8_dbias")


def fp8_dbias_noalloc(g: torch.Tensor, dbias: torch.Tensor, g_scale: torch.Tensor | None = None,
                      g_fmt: int | None = None) -> None:
    """fp8_dbias without a workspace: for callers that cannot allocate device
    memory; its scratch is a fixed 1 MiB array inside the library (calls that
    overlap on the GPU race; the first call on a device should come before any
    stream capture)."""
    M, N = g.shape
    _check(_lib.fp8_dbias_noalloc(_ptr(g), _dtype_code(g, g_fmt), M, N, _ld(g), _ptr(g_scale), _ptr(dbias),
                                  _stream(g.device)), "fp8_dbias_noalloc")


def fp8_linear_forward(args: LinearFwdArgs, device=None) -> None:
    _check(_lib.fp8_linear_forward(ctypes.byref(args), _stream(device)), "fp8_linear_forward")


def fp8_linear_backward(args: LinearBwdArgs, device=None) -> None:
    _check(_lib.fp8_linear_backward(ctypes.byref(args), _stream(device)), "fp8_linear_backward")


def fp8_linear_workspace_bytes(M: int, N: int, K: int) -> int:
    return _lib.fp8_linear_workspace_bytes(M, N, K)


def fp8_get_device_status() -> int:
    return _lib.fp8_get_device_status()


def fp8_wait_selftest(flag: torch.Tensor, limit_ns: int, results: torch.Tensor) -> None:
    """Runs the bounded-wait diagnostic kernel: results[0] / results[1] = 1
    where the flag wait / the mbarrier wait was satisfied, 0 where it ran out
    (which fp8_get_device_status then reports as FP8_ERR_DEVICE_TIMEOUT)."""
    _check(_lib.fp8_wait_selftest(_ptr(flag), limit_ns, _ptr(results), _stream(flag.device)), "fp8_wait_selftest")


def fp8_status_string(status: int) -> str:
    return _lib.fp8_status_string(status).decode()


def fp8_version() -> str:
    return _lib.fp8_version().decode()


# --------------------------------------------------------------------------- helpers

class ScaleRing:
    """Delayed-scaling state of one tensor: a device buffer laid out as
    [hist (H fp32) | scale | step | ticket | scratch]."""

    def __init__(self, hist_len: int = 16, device="cuda", seed_amax: float | None = None, fmt: int = FP8_E4M3,
                 buf: torch.Tensor | None = None):
        self.H = hist_len
        words = fp8_ring_bytes(hist_len) // 4
        if buf is not None:
            if buf.dtype != torch.float32 or buf.numel() != words or not buf.is_contiguous():
                raise ValueError(f"ring buffer must be {words} contiguous fp32 words")
            self.buf = buf
        else:
            self.buf = torch.empty(words, dtype=torch.float32, device=device)
        if seed_amax is None:
            fp8_ring_init(self.buf, hist_len)
        else:
            fp8_ring_seed(self.buf, hist_len, fmt, seed_amax)

    @property
    def hist(self):
        return self.buf[: self.H]

    @property
    def scale(self):
        return self.buf[self.H]

    @property
    def step(self):
        return int(self.buf[self.H + 1 : self.H + 2].view(torch.int32).item())

    def words(self):
        return self.buf.view(torch.int32)


def quantize(x: torch.Tensor, fmt: int, ring: ScaleRing | None, out: torch.Tensor | None = None):
    """Quantize x with its ring (ring None: current scaling from x's own amax);
    returns (codes [rows, cols] uint8 view with a 16-aligned row stride, amax
    (1-elem fp32), scale used (1-elem fp32))."""
    rows, cols = x.shape
    if out is None:
        out = fp8_alloc(rows, cols, x.device)
    amax = torch.empty(1, dtype=torch.float32, device=x.device)
    scale = torch.empty(1, dtype=torch.float32, device=x.device)
    fp8_quantize(x, fmt, ring.buf if ring is not None else None, ring.H if ring is not None else 0, out, amax, scale)
    return out, amax, scale


@dataclass
class ForwardResult:
    y: torch.Tensor
    x8: torch.Tensor
    w8: torch.Tensor
    sx: torch.Tensor
    sw: torch.Tensor
    amax_x: torch.Tensor
    amax_w: torch.Tensor


def linear_forward(x, w, ring_x: ScaleRing | None, ring_w: ScaleRing | None, bias=None, bias_scale=None,
                   fmt_x=FP8_E4M3, fmt_w=FP8_E4M3, x_scale_in=None, w_scale_in=None, hist_len=16,
                   y=None, x8=None, w8=None, scales=None) -> ForwardResult:
    """y = x w^T + bias through fp8_linear_forward.  x/w may be bf16/fp16/fp32
    or fp8 codes (torch.float8_* or uint8 with their fmt, plus *_scale_in).
    scales: optional 4-element fp32 device buffer receiving sx, sw, amax_x,
    amax_w (allocated here when None)."""
    M, K = x.shape
    N = w.shape[0]
    dev = x.device
    xq = x.dtype in (torch.uint8, torch.float8_e4m3fn, torch.float8_e5m2)
    wq = w.dtype in (torch.uint8, torch.float8_e4m3fn, torch.float8_e5m2)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if y is None else y
    if x8 is None:
        x8 = x.view(torch.uint8) if xq else fp8_alloc(M, K, dev)
    if w8 is None:
        w8 = w.view(torch.uint8) if wq else fp8_alloc(N, K, dev)
    sc = torch.empty(4, dtype=torch.float32, device=dev) if scales is None else scales
    H = ring_x.H if ring_x is not None else (ring_w.H if ring_w is not None else hist_len)
    bias_dtype = FP8_DT_BF16
    if bias is not None and bias.dtype != torch.bfloat16:
        bias_dtype = _dtype_code(bias, FP8_E4M3)
    args = LinearFwdArgs(
        M, N, K,
        _ptr(x), _dtype_code(x, fmt_x), _ld(x), _ptr(x_scale_in),
        _ptr(w), _dtype_code(w, fmt_w), _ld(w), _ptr(w_scale_in),
        _ptr(bias), bias_dtype, _ptr(bias_scale),
        fmt_x, fmt_w, H,
        _ptr(ring_x.buf) if ring_x is not None else None, _ptr(ring_w.buf) if ring_w is not None else None,
        _ptr(x8), _ld(x8), _ptr(w8), _ld(w8),
        _ptr(sc[0:1]), _ptr(sc[1:2]), _ptr(sc[2:3]), _ptr(sc[3:4]),
        _ptr(y), _ld(y))
    fp8_linear_forward(args, dev)
    return ForwardResult(y, x8, w8, sc[0:1], sc[1:2], sc[2:3], sc[3:4])


@dataclass
class BackwardResult:
    dx: torch.Tensor | None
    dw: torch.Tensor | None
    dbias: torch.Tensor | None
    g8: torch.Tensor
    sg: torch.Tensor
    amax_g: torch.Tensor


def linear_backward(g, fwd: ForwardResult, ring_g: ScaleRing | None, fmt_g=FP8_E5M2, fmt_x=FP8_E4M3,
                    fmt_w=FP8_E4M3, need_dx=True, need_dw=True, need_dbias=False, g_scale_in=None,
                    workspace=None, dx=None, dw=None, dbias=None, g8=None) -> BackwardResult:
    """dX, dW, dbias through fp8_linear_backward, reusing the forward's x8/w8
    and scale snapshots."""
    M, N = g.shape
    K = fwd.x8.shape[1]
    dev = g.device
    gq = g.dtype in (torch.uint8, torch.float8_e4m3fn, torch.float8_e5m2)
    if g8 is None:
        g8 = g.view(torch.uint8) if gq else fp8_alloc(M, N, dev)
    dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if (need_dx and dx is None) else dx
    dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if (need_dw and dw is None) else dw
    dbias = torch.empty(N, dtype=torch.bfloat16, device=dev) if (need_dbias and dbias is None) else dbias
    if need_dbias and workspace is None:
        workspace = torch.zeros(max(16, fp8_linear_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
    sc = torch.empty(2, dtype=torch.float32, device=dev)
    H = ring_g.H if ring_g is not None else 16
    args = LinearBwdArgs(
        M, N, K,
        _ptr(g), _dtype_code(g, fmt_g), _ld(g), _ptr(g_scale_in),
        fmt_g, H, _ptr(ring_g.buf) if ring_g is not None else None,
        _ptr(g8), _ld(g8), _ptr(sc[0:1]), _ptr(sc[1:2]),
        _ptr(fwd.x8), _ld(fwd.x8), _ptr(fwd.sx), fmt_x,
        _ptr(fwd.w8), _ld(fwd.w8), _ptr(fwd.sw), fmt_w,
        int(need_dx), int(need_dw), int(need_dbias),
        _ptr(dx), _ld(dx) if dx is not None else 0,
        _ptr(dw), _ld(dw) if dw is not None else 0,
        _ptr(dbias),
        _ptr(workspace), (workspace.numel() * workspace.element_size()) if workspace is not None else 0)
    fp8_linear_backward(args, dev)
    return BackwardResult(dx, dw, dbias, g8, sc[0:1], sc[1:2])
