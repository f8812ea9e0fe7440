"""Shared helpers for the GPU parity tests: conversions between torch tensors
and the oracle's numpy bit patterns, padded device buffers, and the GEMM
tolerance check."""
import numpy as np
import torch

import oracle


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16/fp16 tensor -> uint16 bit patterns; fp32 -> float32; uint8 -> uint8 (CPU copies)."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.float8_e4m3fn, torch.float8_e5m2):
        return t.view(torch.uint8).numpy()
    return t.numpy()


def dt_code(t: torch.Tensor) -> int:
    return {torch.bfloat16: oracle.DT_BF16, torch.float16: oracle.DT_FP16, torch.float32: oracle.DT_FP32}[t.dtype]


def padded(t_cpu: torch.Tensor, ld: int, device="cuda") -> torch.Tensor:
    """Copy a 2-D CPU tensor to the device with row stride ld (>= cols); the
    padding holds a large finite junk value, so reading it would change amax
    (or the GEMM result).  Returns the [rows, cols] view."""
    rows, cols = t_cpu.shape
    buf = torch.full((rows, ld), 0x77, dtype=t_cpu.dtype) if t_cpu.dtype == torch.uint8 else \
        torch.full((rows, ld), 30000.0, dtype=t_cpu.dtype)
    buf[:, :cols] = t_cpu
    return buf.to(device)[:, :cols]


def fp8_buffer(rows: int, cols: int, ld: int | None = None, device="cuda", fill=0xA5) -> torch.Tensor:
    ld = (cols + 15) // 16 * 16 if ld is None else ld
    return torch.full((rows, ld), fill, dtype=torch.uint8, device=device)[:, :cols]


def host_rows(t: torch.Tensor) -> np.ndarray:
    """Device [rows, cols] view -> numpy [rows, cols] copy."""
    return t.detach().cpu().contiguous().numpy()


def ring_words(ring) -> np.ndarray:
    return ring.buf.detach().cpu().view(torch.int32).numpy().view(np.uint32)


def oracle_ring_words(r: oracle.Ring) -> np.ndarray:
    w = np.zeros(r.H + 4, np.uint32)
    w[: r.H] = r.hist.view(np.uint32)
    w[r.H] = np.float32(r.scale).view(np.uint32)
    w[r.H + 1] = r.step
    w[r.H + 2] = 0
    w[r.H + 3] = 0
    return w


def assert_codes_equal(got: np.ndarray, want: np.ndarray, fmt: int):
    """fp8 codes equal byte for byte; NaN codes only need to be NaN on both sides."""
    if np.array_equal(got, want):
        return
    nan_w = (want & 0x7F) == 0x7F if fmt == oracle.E4M3 else (want & 0x7F) >= 0x7D
    nan_g = (got & 0x7F) == 0x7F if fmt == oracle.E4M3 else (got & 0x7F) >= 0x7D
    bad = (got != want) & ~(nan_w & nan_g)
    if bad.any():
        idx = np.argwhere(bad)[:8]
        raise AssertionError(f"{bad.sum()} fp8 codes differ, first at {idx.tolist()}: "
                             f"got {got[tuple(idx.T)]} want {want[tuple(idx.T)]}")


def assert_gemm_close(y_gpu_bits: np.ndarray, y_orc_bits: np.ndarray, sumabs: np.ndarray, sa: float, sb: float,
                      what: str = ""):
    """|y_gpu - y_oracle| <= max(1 bf16 ulp of the oracle value, 2e-6 sum|ab| / (sa sb))."""
    g = oracle.bf16_to_f32(y_gpu_bits).astype(np.float64)
    o = oracle.bf16_to_f32(y_orc_bits).astype(np.float64)
    tol = oracle.gemm_tolerance(y_orc_bits, sumabs, sa, sb)
    # non-finite oracle outputs (IEEE fp32 accumulation of NaN / inf operands)
    # must be matched exactly: NaN by NaN, an infinity by the same infinity
    both_nan = np.isnan(g) & np.isnan(o)
    same_inf = np.isinf(o) & (g == o)
    exact = both_nan | same_inf
    with np.errstate(invalid="ignore"):
        err = np.where(exact, 0.0, np.abs(g - o))
    bad = ~((err <= tol) | exact)  # a non-finite output's tolerance is non-finite too
    if bad.any():
        idx = np.argwhere(bad)[:6]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first "
                             f"{[(tuple(i), g[tuple(i)], o[tuple(i)], tol[tuple(i)]) for i in idx]}")
    live = ~exact
    return float(np.max(err[live] / tol[live])) if live.any() else 0.0


def sample_points(rng, I: int, J: int, nrows=64, ncols=64, nrand=4096):
    """Seeded sample of output coordinates: full rows, full columns, random points."""
    rows = rng.choice(I, size=min(nrows, I), replace=False)
    cols = rng.choice(J, size=min(ncols, J), replace=False)
    pi = np.concatenate([np.repeat(rows, J), np.tile(np.arange(I), len(cols)), rng.integers(0, I, nrand)])
    pj = np.concatenate([np.tile(np.arange(J), len(rows)), np.repeat(cols, I), rng.integers(0, J, nrand)])
    return pi.astype(np.int64), pj.astype(np.int64)
