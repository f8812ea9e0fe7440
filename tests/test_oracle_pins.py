"""Pins of the CPU oracle to facts other than itself (CPU only, no GPU).

Each test checks one oracle function against the format definitions, a
library routine, brute force, exact rational arithmetic, a closed form or an
invariant stated by the AstrAI commit-log pages.  The mutant tests at the end
plant plausible mistakes in copies of oracle logic and check that a pin fails.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import DT_BF16, DT_E4M3, DT_E5M2, DT_FP16, DT_FP32, E4M3, E5M2, FP8_MAX

HERE = os.path.dirname(os.path.abspath(__file__))
FMTS = (E4M3, E5M2)
TORCH_F8 = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


# ---------------------------------------------------------------- helpers

def ref_encode(fmt, v32):
    """Independent saturating RNE cast: arithmetic rounding with np.rint on the
    magnitude divided by the quantum of its binade, then the code assembled
    from exponent and mantissa fields.  Written from the OFP8 definition."""
    mbits, bias, emin = (3, 7, -6) if fmt == E4M3 else (2, 15, -14)
    fmax = FP8_MAX[fmt]
    v = np.asarray(v32, np.float32).astype(np.float64)
    out = np.zeros(v.shape, np.uint8)
    nan = np.isnan(v)
    sign = np.signbit(v)
    a = np.where(nan, 0.0, np.abs(v))
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(ex - 1, emin)
    q = np.ldexp(1.0, e - mbits)
    with np.errstate(invalid="ignore"):
        r = np.rint(a / q) * q
    r = np.where(np.isinf(a) | (r > fmax), fmax, r)
    # assemble code from r
    _, ex2 = np.frexp(np.where(r > 0, r, 1.0))
    e2 = ex2 - 1
    sub = r < 2.0 ** emin
    m_sub = np.round(r / 2.0 ** (emin - mbits)).astype(np.int64)
    m_norm = np.round((r / np.ldexp(1.0, e2) - 1.0) * (1 << mbits)).astype(np.int64)
    code = np.where(sub, m_sub, ((e2 + bias) << mbits) | m_norm)
    out = (code.astype(np.int64) & 0x7F).astype(np.uint8) | np.where(sign, 0x80, 0).astype(np.uint8)
    out = np.where(nan, 0x7F, out).astype(np.uint8)
    return out


def is_nan_code(fmt, c):
    c = np.asarray(c).astype(np.int64) & 0x7F
    return (c == 0x7F) if fmt == E4M3 else (c >= 0x7D)


def all_bf16_values():
    bits = np.arange(65536, dtype=np.uint32)
    return (bits << 16).view(np.float32)


def all_fp16_values():
    return np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float32)


def rand_codes(rng, fmt, shape, lo=0x00, hi=None):
    """Random finite fp8 codes (both signs)."""
    hi = (0x7E if fmt == E4M3 else 0x7B) if hi is None else hi
    mag = rng.integers(lo, hi + 1, size=shape)
    sign = rng.integers(0, 2, size=shape) << 7
    return (mag | sign).astype(np.uint8)


# ---------------------------------------------------------------- formats

def test_golden_format_points():
    """Selected codes against values typed from the OFP8 definition."""
    names = {"e4m3": E4M3, "e5m2": E5M2}
    tabs = {f: oracle.decode_table(f) for f in FMTS}
    n = 0
    with open(os.path.join(HERE, "golden", "fp8_format_points.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if not line:
                continue
            f, code, val = line.split()
            got = tabs[names[f]][int(code, 16)]
            want = float(val)
            if math.isnan(want):
                assert math.isnan(got), (f, code)
            else:
                assert got == want and math.copysign(1, got) == math.copysign(1, want), (f, code, got)
            n += 1
    assert n >= 25


@pytest.mark.parametrize("fmt", FMTS)
def test_decode_table_structure(fmt):
    """Non-negative finite codes are strictly increasing, negatives mirror
    them, and the number of finite values matches the definition."""
    t = oracle.decode_table(fmt)
    top = 0x7E if fmt == E4M3 else 0x7B
    pos = t[: top + 1]
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(t[0x80: 0x80 + top + 1], -pos)
    assert pos[-1] == FP8_MAX[fmt]
    finite = np.isfinite(t).sum()
    assert finite == (254 if fmt == E4M3 else 248)


@pytest.mark.parametrize("fmt", FMTS)
def test_decode_matches_torch(fmt):
    """Library special case: torch's float8 dtypes decode every code alike."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    tv = codes.view(TORCH_F8[fmt]).to(torch.float64).numpy()
    ov = oracle.decode_table(fmt)
    nan = np.isnan(ov)
    assert np.array_equal(nan, np.isnan(tv))
    assert np.array_equal(ov[~nan], tv[~nan])


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_roundtrip(fmt):
    t = oracle.decode_table(fmt)
    codes = np.array([c for c in range(256) if np.isfinite(t[c])], np.uint8)
    back = oracle.encode(fmt, t[codes].astype(np.float32))
    assert np.array_equal(back, codes)


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_specials(fmt):
    top = 0x7E if fmt == E4M3 else 0x7B
    v = np.array([np.inf, -np.inf, 1e30, -1e30, FP8_MAX[fmt] * 1.01, np.nan, -0.0, 0.0, -1e-30],
                 np.float32)
    got = oracle.encode(fmt, v)
    assert list(got[:5]) == [top, 0x80 | top, top, 0x80 | top, top]
    assert got[5] == 0x7F
    assert got[6] == 0x80 and got[7] == 0x00 and got[8] == 0x80


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_vs_independent_rounding(fmt):
    """Every bf16 value times several scales (product rounded to fp32 first),
    and every fp16 value: exhaustive scan == arithmetic RNE rounding."""
    vals = [all_bf16_values(), all_fp16_values()]
    for base in vals:
        for s in (1.0, 2.0 ** -7, 3.5, 448.0 / 7.3):
            with np.errstate(over="ignore", invalid="ignore"):
                p = (base * np.float32(s)).astype(np.float32)
            got = oracle.encode(fmt, p)
            want = ref_encode(fmt, p)
            nan = np.isnan(p)
            assert np.array_equal(got[~nan], want[~nan]), (fmt, s)
            assert np.all(is_nan_code(fmt, got[nan]))


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_vs_torch_in_range(fmt):
    """Library special case: torch's CPU cast (RNE, no saturation) agrees for
    |v| <= fp8_max."""
    base = all_bf16_values()
    for s in (1.0, 2.0 ** -7, 3.5):
        with np.errstate(over="ignore", invalid="ignore"):
            p = (base * np.float32(s)).astype(np.float32)
        ok = np.isfinite(p) & (np.abs(p) <= FP8_MAX[fmt])
        p = p[ok]
        tcodes = torch.from_numpy(p).to(TORCH_F8[fmt]).view(torch.uint8).numpy()
        assert np.array_equal(oracle.encode(fmt, p), tcodes)


@pytest.mark.parametrize("fmt", FMTS)
def test_encode_midpoints_tie_to_even(fmt):
    """Every midpoint between adjacent grid values goes to the even code;
    one fp32 ulp either side goes to the nearer value."""
    t = oracle.decode_table(fmt)
    top = 0x7E if fmt == E4M3 else 0x7B
    for c in range(top):
        lo, hi = t[c], t[c + 1]
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2  # midpoints are exact in fp32
        even = c if c % 2 == 0 else c + 1
        assert oracle.encode(fmt, [mid])[0] == even
        assert oracle.encode(fmt, [-mid])[0] == 0x80 | even
        below = np.nextafter(mid, np.float32(-np.inf), dtype=np.float32)
        above = np.nextafter(mid, np.float32(np.inf), dtype=np.float32)
        assert oracle.encode(fmt, [below])[0] == c
        assert oracle.encode(fmt, [above])[0] == c + 1


def test_bf16_rne_vs_torch():
    """Library special case: torch's fp32 -> bf16 cast (RNE) on random values,
    exact ties, and values near the overflow threshold."""
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, size=200000, dtype=np.uint64).astype(np.uint32)
    ties = (rng.integers(0, 2 ** 16, size=20000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    edge = np.array([0x7F7F7FFF, 0x7F7F8000, 0x7F7F8001, 0x7F7FFFFF, 0x00008000, 0x00018000,
                     0x80008000, 0x3F808000, 0x3F818000], np.uint32)
    v = np.concatenate([bits, ties, edge]).view(np.float32)
    v = v[~np.isnan(v)]
    got = oracle.bf16_rne(v)
    want = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- amax / quantize

@pytest.mark.parametrize("dtype", (DT_BF16, DT_FP16, DT_FP32))
def test_amax_definition(dtype):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((37, 53)) * 3).astype(np.float32)
    x[5, 7] = -91.0
    x[3, 3] = np.nan
    if dtype == DT_BF16:
        xt = torch.from_numpy(x).to(torch.bfloat16)
        bits = xt.view(torch.int16).numpy().view(np.uint16)
        ref = np.nanmax(np.abs(xt.float().numpy()))
    elif dtype == DT_FP16:
        bits = x.astype(np.float16).view(np.uint16)
        ref = np.nanmax(np.abs(x.astype(np.float16).astype(np.float32)))
    else:
        bits, ref = x, np.nanmax(np.abs(x))
    assert oracle.amax(bits, dtype) == np.float32(ref) == np.float32(91.0)
    # strided view: only the first 40 columns count
    assert oracle.amax(bits, dtype, cols=5) == np.float32(np.nanmax(np.abs(oracle.to_f32(bits, dtype)[:, :5])))
    assert oracle.amax(np.zeros((0, 4), np.float32), DT_FP32) == 0.0


def test_amax_is_raw_not_quantized():
    """The pages' amax bug: the max of the quantized values pins at ~fp8_max and
    collapses the scale.  With saturation the raw amax exceeds fp8_max / s."""
    x = np.array([[1.0, -3.0, 700.0, 2.0]], np.float32)
    ring = oracle.Ring(16)
    q, a, s = oracle.quantize(x, DT_FP32, E4M3, ring)
    assert a == 700.0 and s == 1.0
    deq = oracle.decode(E4M3, q) / s
    assert np.max(np.abs(deq)) == 448.0 < a
    assert ring.scale == np.float32(448.0) / np.float32(700.0)


def test_quantize_definition_and_padding():
    rng = np.random.default_rng(3)
    x = torch.from_numpy(rng.standard_normal((5, 20)).astype(np.float32)).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    s = np.float32(448.0 / 3.3)
    q = oracle.quantize_codes(bits, DT_BF16, E4M3, s, cols=13, ld_out=32)
    p = (x.float().numpy()[:, :13] * s).astype(np.float32)
    assert np.array_equal(q[:, :13], ref_encode(E4M3, p))
    assert np.all(q[:, 13:] == 0)


# ---------------------------------------------------------------- ring

def closed_form_scale(amaxes, H, fmt, init=1.0):
    """scale after t steps = fp8_max / max of the last min(t, H) amaxes, with the
    keep-old rule when that max is 0 / inf or the quotient overflows."""
    s = np.float32(init)
    for t in range(1, len(amaxes) + 1):
        m = np.float32(max(amaxes[max(0, t - H):t]))
        if m > 0 and np.isfinite(m):
            with np.errstate(over="ignore"):
                q = np.float32(FP8_MAX[fmt]) / m
            if np.isfinite(q):
                s = q
    return s


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("H", (1, 3, 16))
def test_ring_closed_form(fmt, H):
    rng = np.random.default_rng(4 + H)
    amaxes = [np.float32(a) for a in np.exp(rng.uniform(-6, 6, size=41)).astype(np.float32)]
    ring = oracle.Ring(H)
    for t, a in enumerate(amaxes, 1):
        ring.advance(a, fmt)
        assert ring.scale == closed_form_scale(amaxes[:t], H, fmt), t
        assert ring.step == t
        # hist[i] holds the latest a_j with (j-1) % H == i
        for i in range(H):
            js = [j for j in range(1, t + 1) if (j - 1) % H == i]
            assert ring.hist[i] == (amaxes[js[-1] - 1] if js else 0.0)


def test_ring_keep_old_rules():
    ring = oracle.Ring(4)
    ring.seed(2.0, E4M3)
    assert ring.scale == np.float32(224.0)
    ring.advance(0.0, E4M3)
    assert ring.scale == np.float32(224.0)  # window max 0 -> keep
    ring.advance(np.inf, E4M3)
    assert ring.scale == np.float32(224.0)  # window max inf -> keep
    r2 = oracle.Ring(2)
    r2.advance(1e-40, E5M2)                # 57344 / 1e-40 overflows fp32 -> keep
    assert r2.scale == 1.0
    r2.advance(8.0, E5M2)
    assert r2.scale == np.float32(57344.0 / 8.0)
    r3 = oracle.Ring(3)
    r3.seed(0.0, E4M3)
    assert r3.scale == 1.0


# ---------------------------------------------------------------- GEMM

def frac_dot(avals, bvals):
    return sum((Fraction(float(x)) * Fraction(float(y)) for x, y in zip(avals, bvals)), Fraction(0))


@pytest.mark.parametrize("fa,fb", ((E4M3, E4M3), (E5M2, E4M3), (E5M2, E5M2)))
def test_gemm_exact_rational(fa, fb):
    """Tiny shapes: the exact path equals the rational dot (rounded once), the
    fp32 path is within K * 2^-24 * sum|ab| of it, sum|ab| (double, only a
    tolerance input) is within K * 2^-53 relative of the rational sum, for the
    forward, dX and dW operand layouts written out with explicit indices."""
    rng = np.random.default_rng(5)
    ta, tb = oracle.decode_table(fa), oracle.decode_table(fb)
    for (M, N, K) in ((3, 4, 5), (2, 3, 37), (4, 1, 64)):
        a = rand_codes(rng, fa, (M, K))        # X8 / G8 role
        b = rand_codes(rng, fb, (N, K))        # W8 role
        acc, ex, sab = oracle.gemm_acc(a, fa, K, 1, b, fb, K, 1, M, N, K, exact=True)
        for i in range(M):
            for j in range(N):
                fr = frac_dot(ta[a[i]], tb[b[j]])
                assert ex[i, j] == float(fr)
                sa = sum(abs(Fraction(float(x)) * Fraction(float(y))) for x, y in zip(ta[a[i]], tb[b[j]]))
                assert abs(Fraction(float(sab[i, j])) - sa) <= Fraction(K) * Fraction(2) ** -53 * sa
                assert abs(Fraction(float(acc[i, j])) - fr) <= Fraction(K) * Fraction(2) ** -24 * sa
        # dX layout: dX[m,k] = sum_n G[m,n] W[n,k]; G is a [M,K'] with K' = contraction
        g = rand_codes(rng, fa, (M, N))
        w = rand_codes(rng, fb, (N, K))
        acc, ex, _ = oracle.dx_acc(g, N, fa, w, K, fb, M, N, K, exact=True)
        for m in range(M):
            for k in range(K):
                assert ex[m, k] == float(frac_dot(ta[g[m, :]], tb[w[:, k]]))
        # dW layout: dW[n,k] = sum_m G[m,n] X[m,k]
        x = rand_codes(rng, fb, (M, K))
        acc, ex, _ = oracle.dw_acc(g, N, fa, x, K, fb, M, N, K, exact=True)
        for n in range(N):
            for k in range(K):
                assert ex[n, k] == float(frac_dot(ta[g[:, n]], tb[x[:, k]]))


def test_gemm_small_integer_exact():
    """fp8 values that are small integers: every partial sum is an integer below
    2^24, so the fp32 result equals the integer matmul exactly."""
    rng = np.random.default_rng(6)
    t = oracle.decode_table(E4M3)
    int_codes = np.array([c for c in range(256) if np.isfinite(t[c]) and t[c] == np.round(t[c])
                          and abs(t[c]) <= 16], np.uint8)
    M, N, K = 16, 24, 200
    a = rng.choice(int_codes, size=(M, K))
    b = rng.choice(int_codes, size=(N, K))
    acc, _, _ = oracle.fwd_acc(a, K, E4M3, b, K, E4M3, M, N, K)
    ref = t[a].astype(np.int64) @ t[b].astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), ref)


def test_gemm_identity_weight():
    """W8 = identity (code 0x38 = 1.0): Y = bf16(decode(x8) / sx) exactly (as
    values: a -0 input gives +0, the fp32 sum starting from +0)."""
    rng = np.random.default_rng(7)
    M, K = 8, 48
    x8 = rand_codes(rng, E4M3, (M, K))
    w8 = np.where(np.eye(K, dtype=bool), 0x38, 0x00).astype(np.uint8)
    sx = np.float32(448.0 / 3.7)
    acc, _, _ = oracle.fwd_acc(x8, K, E4M3, w8, K, E4M3, M, K, K)
    y, _ = oracle.epilogue(acc, sx, 1.0)
    want = (torch.from_numpy(oracle.decode(E4M3, x8).astype(np.float32)) / float(sx)).to(torch.bfloat16)
    assert np.array_equal(oracle.bf16_to_f32(y), want.float().numpy())


def test_gemm_vs_float64_matmul():
    """Random c1-sized operands: fp32 result vs numpy's float64 matmul of the
    decoded values, within K * 2^-24 * sum|ab|."""
    rng = np.random.default_rng(8)
    M, N, K = 64, 192, 128
    a = rand_codes(rng, E4M3, (M, K))
    b = rand_codes(rng, E4M3, (N, K))
    acc, ex, sab = oracle.fwd_acc(a, K, E4M3, b, K, E4M3, M, N, K, exact=True)
    ref = oracle.decode(E4M3, a) @ oracle.decode(E4M3, b).T
    assert np.all(np.abs(acc - ref) <= K * 2.0 ** -24 * sab)
    assert np.all(np.abs(ex - ref) <= 2.0 ** -40 * sab)


def test_layouts_match_transposed_copies():
    """dX and dW read transposed operands through strides; they must equal the
    forward routine run on explicitly transposed copies (same k order)."""
    rng = np.random.default_rng(9)
    M, N, K = 20, 12, 28
    g8 = rand_codes(rng, E5M2, (M, N))
    w8 = rand_codes(rng, E4M3, (N, K))
    x8 = rand_codes(rng, E4M3, (M, K))
    dx, _, _ = oracle.dx_acc(g8, N, E5M2, w8, K, E4M3, M, N, K)
    dx2, _, _ = oracle.fwd_acc(g8, N, E5M2, np.ascontiguousarray(w8.T), N, E4M3, M, K, N)
    assert np.array_equal(dx, dx2)
    dw, _, _ = oracle.dw_acc(g8, N, E5M2, x8, K, E4M3, M, N, K)
    dw2, _, _ = oracle.fwd_acc(np.ascontiguousarray(g8.T), M, E5M2, np.ascontiguousarray(x8.T), M,
                               E4M3, N, K, M)
    assert np.array_equal(dw, dw2)
    assert not np.array_equal(dw, dw2.T[:N, :K]) if N == K else True


def test_epilogue_bias_fused_vs_split():
    """Fused bias (one bf16 rounding) is within 1 bf16 ulp of the split path
    (round, add, round) for the pages' bias distribution N(0, 0.01) (astrai
    @4019dda, fused-bias bullet), is always at least as close to the float64
    value, and an fp8 bias is decode(b8) / bias_scale."""
    rng = np.random.default_rng(10)
    acc = (rng.standard_normal((64, 96)) * 50).astype(np.float32)
    sa, sb = np.float32(3.0), np.float32(0.75)
    nob, _ = oracle.epilogue(acc, sa, sb)
    for bstd in (0.01, 0.7):
        bias = torch.from_numpy((rng.standard_normal(96) * bstd).astype(np.float32)).to(torch.bfloat16)
        bbits = bias.view(torch.int16).numpy().view(np.uint16)
        fused, ffused = oracle.epilogue(acc, sa, sb, bbits, DT_BF16)
        split = oracle.bf16_rne(oracle.bf16_to_f32(nob) + bias.float().numpy()[None, :])
        f_fused = oracle.bf16_to_f32(fused).astype(np.float64)
        f_split = oracle.bf16_to_f32(split).astype(np.float64)
        exact = acc.astype(np.float64) / (float(sa) * float(sb)) + bias.double().numpy()[None, :]
        if bstd == 0.01:
            ulp = np.maximum(oracle.bf16_ulp(f_fused), oracle.bf16_ulp(f_split))
            assert np.all(np.abs(f_fused - f_split) <= ulp)
        assert np.all(np.abs(f_fused - exact) <= 0.5 * oracle.bf16_ulp(exact) * (1 + 2.0 ** -20) + 1e-6 * np.abs(exact))
        assert np.all(np.abs(f_fused - exact) <= np.abs(f_split - exact) + 1e-6 * np.abs(exact))
        assert np.array_equal(ffused, (acc / (sa * sb) + bias.float().numpy()[None, :]).astype(np.float32))
    # fp8 bias
    b8 = rand_codes(rng, E4M3, (96,))
    bsc = np.float32(448.0 / 2.5)
    _, f8 = oracle.epilogue(acc, sa, sb, b8, DT_E4M3, bsc)
    bv = (oracle.decode(E4M3, b8).astype(np.float32) / bsc).astype(np.float32)
    assert np.array_equal(f8, (acc / (sa * sb) + bv[None, :]).astype(np.float32))


# ---------------------------------------------------------------- dbias

def test_dbias():
    rng = np.random.default_rng(11)
    M, N = 300, 70
    gi = rng.integers(-20, 21, size=(M, N)).astype(np.float32)
    gb = torch.from_numpy(gi).to(torch.bfloat16)
    out, f, _ = oracle.dbias(gb.view(torch.int16).numpy().view(np.uint16), DT_BF16, M, N)
    assert np.array_equal(f, gi.sum(0))  # small integers: exact
    gr = torch.from_numpy((rng.standard_normal((M, N)) * 1e-3).astype(np.float32)).to(torch.bfloat16)
    out, f, sa = oracle.dbias(gr.view(torch.int16).numpy().view(np.uint16), DT_BF16, M, N)
    ref = gr.double().numpy().sum(0)
    assert np.all(np.abs(f - ref) <= M * 2.0 ** -24 * sa)
    assert np.array_equal(out, torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    # fp8 g: dequantize each element first
    g8 = rand_codes(rng, E5M2, (M, N), hi=0x50)
    sg = np.float32(3.0)
    _, f8, _ = oracle.dbias(g8, DT_E5M2, M, N, sg)
    deq = (oracle.decode(E5M2, g8).astype(np.float32) / sg).astype(np.float32)
    want = np.zeros(N, np.float32)
    for m in range(M):
        want = (want + deq[m]).astype(np.float32)
    assert np.array_equal(f8, want)


# ---------------------------------------------------------------- orchestration

def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def test_prequantized_weight_skips_quantize():
    """A pre-quantized w8 skips its quantize: amax_w = 0, sw = the caller's
    scale, ring_w untouched."""
    rng = np.random.default_rng(12)
    M, N, K = 8, 16, 32
    x = _bits(_bf16(rng.standard_normal((M, K))))
    w8 = rand_codes(rng, E4M3, (N, K), hi=0x60)
    rx, rw = oracle.Ring(16), oracle.Ring(16)
    rw.seed(5.0, E4M3)
    before = rw.copy()
    out = oracle.linear_forward(M, N, K, x, DT_BF16, w8, DT_E4M3, rx, rw, w_scale_in=2.5)
    assert out["amax_w"] == 0.0 and out["sw"] == np.float32(2.5)
    assert rw.step == before.step and np.array_equal(rw.hist, before.hist) and rw.scale == before.scale
    assert rx.step == 1
    acc, _, _ = oracle.fwd_acc(out["x8"], K, E4M3, w8, K, E4M3, M, N, K)
    y, _ = oracle.epilogue(acc, out["sx"], 2.5)
    assert np.array_equal(y, out["y"])


def test_snapshot_and_backward_scale_reuse():
    """The forward dequantizes with the scale used to quantize (read before the
    ring publishes the next one); the backward reuses the forward's sx, sw."""
    rng = np.random.default_rng(13)
    M, N, K = 16, 24, 32
    rx, rw, rg = oracle.Ring(16), oracle.Ring(16), oracle.Ring(16)
    rx.seed(2.0, E4M3); rw.seed(0.5, E4M3); rg.seed(1e-3, E5M2)
    x = _bits(_bf16(rng.standard_normal((M, K))))
    w = _bits(_bf16(rng.standard_normal((N, K)) * 0.2))
    sx0, sw0 = rx.scale, rw.scale
    f = oracle.linear_forward(M, N, K, x, DT_BF16, w, DT_BF16, rx, rw)
    assert f["sx"] == sx0 and f["sw"] == sw0
    assert rx.scale != sx0 and rw.scale != sw0          # rings moved on
    g = _bits(_bf16(rng.standard_normal((M, N)) * 1e-3))
    sg0 = rg.scale
    b = oracle.linear_backward(M, N, K, g, DT_BF16, rg, f["x8"], E4M3, f["sx"], f["w8"], E4M3, f["sw"],
                               need_dbias=True)
    assert b["sg"] == sg0
    g8 = oracle.quantize_codes(g, DT_BF16, E5M2, sg0)
    assert np.array_equal(b["g8"], g8)
    acc, _, _ = oracle.dx_acc(g8, N, E5M2, f["w8"], K, E4M3, M, N, K)
    assert np.array_equal(b["dx"], oracle.epilogue(acc, sg0, sw0)[0])
    acc, _, _ = oracle.dw_acc(g8, N, E5M2, f["x8"], K, E4M3, M, N, K)
    assert np.array_equal(b["dw"], oracle.epilogue(acc, sg0, sx0)[0])


def test_no_scale_ratio_leak():
    """Two delayed steps where the input amax doubles: the second step's Y must
    match the float64 GEMM of the unquantized inputs within fp8 noise, not be
    off by the scale ratio (astrai/extension/ops @057c0d3 regression)."""
    rng = np.random.default_rng(14)
    M, N, K = 64, 192, 128
    rx, rw = oracle.Ring(16), oracle.Ring(16)
    w = _bf16(rng.standard_normal((N, K)) * 0.02)
    for step in range(3):
        xt = _bf16(rng.standard_normal((M, K)) * 2.0 ** step)
        f = oracle.linear_forward(M, N, K, _bits(xt), DT_BF16, _bits(w), DT_BF16, rx, rw)
        y = oracle.bf16_to_f32(f["y"]).astype(np.float64)
        ref = xt.double().numpy() @ w.double().numpy().T
        rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
        # step 0 starts from scale 1 (coarse); later steps use the delayed scale.
        # E4M3 has 3 mantissa bits; saturation of the top values bounds the error
        # well below the 2x a leaked ratio would give.
        assert rel < 0.25, (step, rel)
        ratio = np.dot(y.ravel(), ref.ravel()) / np.dot(ref.ravel(), ref.ravel())
        assert 0.8 < ratio < 1.2, (step, ratio)


# ---------------------------------------------------------------- dynamic (current) scaling

def test_dynamic_scale_worked_values():
    """amax 3.5 -> s = 448 / 3.5 = 128 exactly; codes of +-3.5, 1.75, 0.5
    are the grid points 448, 224, 64 (all exact powers-of-two multiples)."""
    x = torch.tensor([[3.5, -3.5, 1.75, 0.5, 0.0, -0.0]], dtype=torch.bfloat16)
    q, a, s = oracle.quantize_dynamic(_bits(x), DT_BF16, E4M3)
    assert a == np.float32(3.5) and s == np.float32(128.0)
    v = oracle.decode(E4M3, q[0])
    assert list(v[:5]) == [448.0, -448.0, 224.0, 64.0, 0.0] and np.signbit(v[5])
    q5, a5, s5 = oracle.quantize_dynamic(_bits(x), DT_BF16, E5M2)
    assert s5 == np.float32(57344.0 / 3.5)


@pytest.mark.parametrize("fmt", FMTS)
def test_dynamic_scale_maps_amax_to_fp8_max(fmt):
    """The element of largest magnitude lands on the format's largest finite
    code (fp32 rounding of x*s can only nudge it to the saturated maximum)."""
    rng = np.random.default_rng(40 + fmt)
    for std in (1e-3, 1.0, 300.0):
        x = _bf16(rng.standard_normal((37, 51)) * std)
        q, a, s = oracle.quantize_dynamic(_bits(x), DT_BF16, fmt)
        xf = x.float().numpy()
        i = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
        assert abs(oracle.decode(fmt, q[i[0], i[1]:i[1] + 1])[0]) == FP8_MAX[fmt]
        assert a == np.float32(np.abs(xf).max())
        # every other code stays inside the grid (no saturation beyond amax)
        assert np.all(np.abs(oracle.decode(fmt, q)) <= FP8_MAX[fmt])


def test_dynamic_scale_keep_rules():
    """amax 0 (all zeros / all NaN), inf, or an overflowing quotient -> 1.0."""
    z = np.zeros((2, 8), np.float32)
    assert oracle.quantize_dynamic(z, DT_FP32, E4M3)[2] == 1.0
    n = np.full((2, 8), np.nan, np.float32)
    qn, an, sn = oracle.quantize_dynamic(n, DT_FP32, E4M3)
    assert an == 0.0 and sn == 1.0 and np.all((qn & 0x7F) == 0x7F)
    inf = np.array([[1.0, np.inf]], np.float32)
    assert oracle.quantize_dynamic(inf, DT_FP32, E5M2)[2] == 1.0
    tiny = np.array([[1e-40, 0.0]], np.float32)  # 57344 / 1e-40 overflows fp32
    assert oracle.quantize_dynamic(tiny, DT_FP32, E5M2)[2] == 1.0


def test_dynamic_linear_has_no_saturation_and_no_ring():
    """With ring None the forward uses each operand's own amax: unlike the
    delayed path's first step (scale 1, x ~ 2^step saturating), no element
    saturates except at the amax, and Y tracks the float64 GEMM."""
    rng = np.random.default_rng(41)
    M, N, K = 64, 192, 128
    x = _bf16(rng.standard_normal((M, K)) * 1e3)
    w = _bf16(rng.standard_normal((N, K)) * 0.02)
    f = oracle.linear_forward(M, N, K, _bits(x), DT_BF16, _bits(w), DT_BF16, None, None)
    assert f["sx"] == oracle.dynamic_scale(f["amax_x"], E4M3)
    assert f["sw"] == oracle.dynamic_scale(f["amax_w"], E4M3)
    # codes at the maximum come only from |x| s at or above 432, the midpoint
    # to the next grid value 416 (RNE), never from saturation of larger values
    sat = np.abs(oracle.decode(E4M3, f["x8"])) == 448.0
    prod = (np.abs(x.float().numpy()) * f["sx"]).astype(np.float32)
    assert sat.any() and np.all(prod[sat] >= 432.0) and np.all(prod <= np.float32(448.0) * (1 + 2.0 ** -23))
    y = oracle.bf16_to_f32(f["y"]).astype(np.float64)
    ref = x.double().numpy() @ w.double().numpy().T
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 0.1


def test_mutant_dynamic_scale_from_quantized_max_is_caught():
    """A dynamic path that measured amax after a scale-1 cast (saturating at
    448) would give s = 1 for |x| >> 448: the worked-value pin above rejects
    any s other than fp8_max / raw amax."""
    x = torch.tensor([[5000.0, 1.0]], dtype=torch.bfloat16)
    raw = oracle.amax(_bits(x), DT_BF16)
    q1 = oracle.quantize_codes(_bits(x), DT_BF16, E4M3, np.float32(1.0))
    wrong = oracle.dynamic_scale(np.abs(oracle.decode(E4M3, q1)).max(), E4M3)
    assert wrong != oracle.quantize_dynamic(_bits(x), DT_BF16, E4M3)[2]
    assert oracle.quantize_dynamic(_bits(x), DT_BF16, E4M3)[2] == np.float32(448.0) / raw


# ---------------------------------------------------------------- mutants

def test_mutant_window_without_current_amax_is_caught():
    """A ring that reduces the window before folding the new amax in fails the
    closed form at some step (the per-step check of test_ring_closed_form)."""
    amaxes = [np.float32(v) for v in (1.0, 8.0, 2.0)]
    H = 16
    hist = np.zeros(H, np.float32)
    s = np.float32(1.0)
    differs = []
    for t, a in enumerate(amaxes):
        m = hist.max()                      # planted: max taken before the fold
        hist[t % H] = a
        if m > 0:
            s = np.float32(448.0) / m
        differs.append(s != closed_form_scale(amaxes[: t + 1], H, E4M3))
    assert any(differs)


def test_mutant_quantized_amax_is_caught():
    """amax taken on the quantized values (the pages' old bug) disagrees with
    the oracle's amax when values saturate."""
    x = np.array([[1.0, -3.0, 700.0, 2.0]], np.float32)
    q = oracle.quantize_codes(x, DT_FP32, E4M3, 1.0)
    bad = np.max(np.abs(oracle.decode(E4M3, q)))
    assert bad != oracle.amax(x, DT_FP32)


def test_mutant_transposed_operand_is_caught():
    """Reading W8 with swapped strides in dX gives a different result than the
    transposed-copy check (non-square, non-symmetric operands)."""
    rng = np.random.default_rng(15)
    M, N, K = 6, 10, 10
    g8 = rand_codes(rng, E5M2, (M, N))
    w8 = rand_codes(rng, E4M3, (N, K))
    good, _, _ = oracle.fwd_acc(g8, N, E5M2, np.ascontiguousarray(w8.T), N, E4M3, M, K, N)
    bad, _, _ = oracle.gemm_acc(g8, E5M2, N, 1, w8, E4M3, K, 1, M, K, N)  # planted: W not transposed
    assert not np.array_equal(good, bad)


def test_mutant_ties_away_is_caught():
    """A cast that breaks ties away from zero fails the midpoint pin."""
    t = oracle.decode_table(E4M3)
    mids = np.array([(t[c] + t[c + 1]) / 2 for c in range(0x7D)], np.float32)
    away = np.array([c + 1 for c in range(0x7D)], np.uint8)   # planted rule
    assert not np.array_equal(oracle.encode(E4M3, mids), away)
