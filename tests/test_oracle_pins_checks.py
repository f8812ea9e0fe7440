"""Pins of the oracle parts the parity checks lean on (CPU only, no GPU):

* ``orc_gemm_points`` -- the sampled GEMM behind every large-shape check --
  against the full ``orc_gemm`` for all three operand layouts, against exact
  rational dot products, and on non-finite operands;
* ``bf16_ulp`` and ``gemm_tolerance`` -- the tolerance itself -- against the
  spacing read off the bf16 bit patterns of every bf16 value, and on worked
  values;
* ``orc_fp16_to_f32`` -- the fp16 input decode of amax and quantize -- against
  numpy's IEEE binary16 over all 65,536 codes.

Each group ends with a planted mistake (a swapped stride, an exponent off by
one, a subnormal scale off by one) that one of its pins rejects.
"""
import ctypes
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import E4M3, E5M2

FMTS = (E4M3, E5M2)


def rand_codes(rng, fmt, shape):
    """Random finite fp8 codes of both signs."""
    hi = 0x7E if fmt == E4M3 else 0x7B
    mag = rng.integers(0, hi + 1, size=shape)
    return (mag | (rng.integers(0, 2, size=shape) << 7)).astype(np.uint8)


def layouts(rng, fa, fb, I, J, Kc):
    """The forward, dX and dW operand layouts of one (I, J, Kc) contraction,
    as (name, a, a_si, a_sk, b, b_sj, b_sk) with contiguous storage:
    fwd  A = X8 [I, Kc],  B = W8 [J, Kc]   (both K-major)
    dX   A = G8 [I, Kc],  B = W8 [Kc, J]   (B MN-major)
    dW   A = G8 [Kc, I],  B = X8 [Kc, J]   (both MN-major)."""
    out = []
    a = rand_codes(rng, fa, (I, Kc)); b = rand_codes(rng, fb, (J, Kc))
    out.append(("fwd", a, Kc, 1, b, Kc, 1))
    a = rand_codes(rng, fa, (I, Kc)); b = rand_codes(rng, fb, (Kc, J))
    out.append(("dx", a, Kc, 1, b, 1, J))
    a = rand_codes(rng, fa, (Kc, I)); b = rand_codes(rng, fb, (Kc, J))
    out.append(("dw", a, 1, I, b, 1, J))
    return out


# ---------------------------------------------------------------- sampled GEMM

@pytest.mark.parametrize("fa,fb", ((E4M3, E4M3), (E5M2, E4M3), (E5M2, E5M2)))
def test_gemm_points_equal_full_gemm(fa, fb):
    """Every (i, j) of odd-sized problems, in a shuffled order with repeats:
    the sampled routine's fp32 accumulator is bit-identical to the full one's
    and its sum |ab| equal, for all three layouts."""
    rng = np.random.default_rng(101)
    I, J, Kc = 37, 29, 53
    for name, a, asi, ask, b, bsj, bsk in layouts(rng, fa, fb, I, J, Kc):
        acc, _, sab = oracle.gemm_acc(a, fa, asi, ask, b, fb, bsj, bsk, I, J, Kc)
        ii, jj = np.meshgrid(np.arange(I), np.arange(J), indexing="ij")
        ii, jj = ii.ravel(), jj.ravel()
        perm = rng.permutation(ii.size)
        ii = np.concatenate([ii[perm], ii[:50]])
        jj = np.concatenate([jj[perm], jj[:50]])
        pacc, psab = oracle.gemm_acc_points(ii, jj, a, fa, asi, ask, b, fb, bsj, bsk, Kc)
        assert np.array_equal(pacc.view(np.uint32), acc[ii, jj].view(np.uint32)), name
        assert np.array_equal(psab, sab[ii, jj]), name


def test_gemm_points_exact_rational():
    """Tiny problems against Fraction dots written with explicit indices:
    small-integer operands (every partial sum an integer below 2^24) match
    exactly; random operands stay within Kc 2^-24 sum|ab| of the exact dot and
    sum|ab| within Kc 2^-53 of the exact sum."""
    rng = np.random.default_rng(102)
    t4, t5 = oracle.decode_table(E4M3), oracle.decode_table(E5M2)
    ints = np.array([c for c in range(256) if np.isfinite(t4[c]) and t4[c] == np.round(t4[c]) and abs(t4[c]) <= 16],
                    np.uint8)
    I, J, Kc = 5, 4, 23
    a = rng.choice(ints, size=(Kc, I))          # dW layout: A MN-major
    b = rng.choice(ints, size=(Kc, J))
    ii = np.repeat(np.arange(I), J)
    jj = np.tile(np.arange(J), I)
    acc, _ = oracle.gemm_acc_points(ii, jj, a, E4M3, 1, I, b, E4M3, 1, J, Kc)
    for t in range(ii.size):
        want = sum(Fraction(float(t4[a[k, ii[t]]])) * Fraction(float(t4[b[k, jj[t]]])) for k in range(Kc))
        assert Fraction(float(acc[t])) == want
    a = rand_codes(rng, E5M2, (I, Kc))          # dX layout: A K-major, B MN-major
    b = rand_codes(rng, E4M3, (Kc, J))
    acc, sab = oracle.gemm_acc_points(ii, jj, a, E5M2, Kc, 1, b, E4M3, 1, J, Kc)
    for t in range(ii.size):
        terms = [Fraction(float(t5[a[ii[t], k]])) * Fraction(float(t4[b[k, jj[t]]])) for k in range(Kc)]
        exact, sa = sum(terms, Fraction(0)), sum((abs(x) for x in terms), Fraction(0))
        assert abs(Fraction(float(acc[t])) - exact) <= Kc * Fraction(2) ** -24 * sa
        assert abs(Fraction(float(sab[t])) - sa) <= Kc * Fraction(2) ** -53 * sa


def ieee_dot_f32(av, bv):
    """sum_k a_k b_k with numpy float32 arithmetic in k order (IEEE: inf and NaN
    propagate, inf * 0 and inf - inf are NaN)."""
    acc = np.float32(0.0)
    with np.errstate(invalid="ignore", over="ignore"):
        for x, y in zip(av, bv):
            acc = np.float32(acc + np.float32(np.float64(x) * np.float64(y)))
    return acc


@pytest.mark.parametrize("case", ["nan", "pinf", "ninf", "inf_times_zero", "both_infs"])
def test_gemm_nonfinite_operands_follow_ieee_fp32(case):
    """Non-finite fp8 operands (E5M2 +-inf 0x7C/0xFC, NaN 0x7E; E4M3 NaN 0x7F):
    the full GEMM and the sampled points give what IEEE fp32 arithmetic gives
    (numpy float32, k order) -- NaN, +-inf -- at the outputs that read them,
    with the sum of magnitudes non-finite there too; every other output is
    unchanged and finite."""
    rng = np.random.default_rng(103)
    I, J, Kc = 6, 5, 40
    a = rand_codes(rng, E5M2, (I, Kc))
    b = rand_codes(rng, E4M3, (J, Kc))
    b[b == 0x80] = 0x08  # no zero operands except the planted one
    b[b == 0x00] = 0x08
    if case == "nan":
        a[2, 17] = 0x7E
    elif case == "pinf":
        a[2, 17] = 0x7C
    elif case == "ninf":
        a[2, 17] = 0xFC
    elif case == "inf_times_zero":
        a[2, 17] = 0x7C
        b[3, 17] = 0x00          # (2, 3): inf * 0
    else:
        a[2, 17], a[2, 30] = 0x7C, 0xFC
        b[:, 17] = b[:, 30] = 0x38  # 1.0: the two infinite products have opposite signs
    acc, ex, sab = oracle.gemm_acc(a, E5M2, Kc, 1, b, E4M3, Kc, 1, I, J, Kc, exact=True)
    ii = np.repeat(np.arange(I), J)
    jj = np.tile(np.arange(J), I)
    pacc, psab = oracle.gemm_acc_points(ii, jj, a, E5M2, Kc, 1, b, E4M3, Kc, 1, Kc)
    da, db = oracle.decode(E5M2, a), oracle.decode(E4M3, b)
    for i in range(I):
        for j in range(J):
            want = ieee_dot_f32(da[i], db[j])
            got = acc[i, j]
            if i == 2:
                assert not np.isfinite(want)
                assert (np.isnan(want) and np.isnan(got)) or want == got, (case, i, j, got, want)
                assert not np.isfinite(sab[i, j]) and not np.isfinite(ex[i, j])
            else:
                assert np.isfinite(got) and np.isfinite(sab[i, j])
    if case == "inf_times_zero":
        assert np.isnan(acc[2, 3]) and np.isinf(acc[2, 0])
    if case == "both_infs":
        assert np.all(np.isnan(acc[2]))
    assert np.array_equal(pacc, acc[ii, jj], equal_nan=True)
    assert np.array_equal(np.isfinite(psab), np.isfinite(sab[ii, jj]))


def test_mutant_points_with_swapped_strides_is_caught():
    """A sampled check that read the dW operand A with its two strides swapped
    (A(i,k) = a[i*I + k] instead of a[k*I + i]) disagrees with the full GEMM."""
    rng = np.random.default_rng(104)
    I, J, Kc = 12, 9, 12                         # square A storage: the swap stays in bounds
    a = rand_codes(rng, E5M2, (Kc, I))
    b = rand_codes(rng, E4M3, (Kc, J))
    acc, _, _ = oracle.gemm_acc(a, E5M2, 1, I, b, E4M3, 1, J, I, J, Kc)
    ii = np.repeat(np.arange(I), J)
    jj = np.tile(np.arange(J), I)
    bad, _ = oracle.gemm_acc_points(ii, jj, a, E5M2, I, 1, b, E4M3, 1, J, Kc)   # planted swap
    assert not np.array_equal(bad, acc[ii, jj])


# ---------------------------------------------------------------- tolerance

def all_bf16_positive_finite():
    """Bit patterns 0x0000 .. 0x7F7F (zero, subnormals, normals up to the
    largest finite bf16) and their values."""
    b = np.arange(0x7F80, dtype=np.uint32)
    return b, (b << 16).view(np.float32)


def spacing_from_bits():
    """Distance from each non-negative finite bf16 value to the next bf16 above
    it, from the bit patterns (consecutive patterns are consecutive values);
    for the largest finite value, where the next pattern is inf, the spacing of
    its binade 2^(127-7)."""
    b, v = all_bf16_positive_finite()
    nxt = ((b + 1) << 16).view(np.float32).astype(np.float64)
    sp = nxt - v.astype(np.float64)
    sp[-1] = 2.0 ** 120
    return v, sp


def test_bf16_ulp_is_the_bit_pattern_spacing():
    """bf16_ulp over every non-negative finite bf16 value (zero, the 127
    subnormals, every normal binade up to the top) equals the gap to the next
    bf16, and is the same for the negated values."""
    v, sp = spacing_from_bits()
    got = oracle.bf16_ulp(v.astype(np.float64))
    assert np.array_equal(got, sp)
    assert np.array_equal(oracle.bf16_ulp(-v.astype(np.float64)), sp)
    assert oracle.bf16_ulp(np.float64(0.0)) == 2.0 ** -133


def test_gemm_tolerance_worked_values():
    """max(1 bf16 ulp of the oracle value, 2e-6 sum|ab| / (sa sb)) on values
    worked by hand: 1.0 has ulp 2^-7, 3.0 has 2^-6, -0.375 has 2^-9, 0 has the
    subnormal spacing 2^-133; sum|ab| = 1e6 with sa sb = 8 gives 0.25."""
    y = oracle.bf16_rne(np.array([1.0, 3.0, -0.375, 0.0, 1.0, 3.0], np.float32))
    sab = np.array([0.0, 0.0, 0.0, 0.0, 1e6, 1e3], np.float64)
    tol = oracle.gemm_tolerance(y, sab, 2.0, 4.0)
    assert np.array_equal(tol[:4], [2.0 ** -7, 2.0 ** -6, 2.0 ** -9, 2.0 ** -133])
    assert abs(tol[4] - 0.25) <= 1e-15 and tol[5] == 2.0 ** -6    # 2e-6 * 1e3 / 8 < ulp(3)
    # unit scales (the bias-gradient form, 2e-6 sum|g|): 2.0 beats ulp(1.0)
    tol1 = oracle.gemm_tolerance(y, sab, 1.0, 1.0)
    assert abs(tol1[4] - 2.0) <= 1e-15 and tol1[5] == 2.0 ** -6


@pytest.mark.parametrize("shift", (-1, +1))
def test_mutant_ulp_exponent_off_by_one_is_caught(shift):
    """A ulp computed one binade off (2^(e-7 +- 1)) fails the spacing pin."""
    v, sp = spacing_from_bits()
    a = v.astype(np.float64)
    with np.errstate(divide="ignore"):
        e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -126.0)
    bad = np.where(a > 0, np.ldexp(1.0, (e - 7 + shift).astype(np.int64)), 2.0 ** -133)   # planted
    assert not np.array_equal(bad, sp)


# ---------------------------------------------------------------- fp16 decode

def fp16_decode_all(fn):
    return np.array([fn(ctypes.c_uint16(h)) for h in range(65536)], np.float32)


def test_fp16_decode_matches_ieee_binary16():
    """orc_fp16_to_f32 over all 65,536 codes against numpy's binary16
    (subnormals, both zeros, infinities; NaN codes give NaN)."""
    got = fp16_decode_all(oracle.lib().orc_fp16_to_f32)
    want = np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))   # signed zeros too
    assert nan.sum() == 2 * 1023


def test_mutant_fp16_subnormal_scale_is_caught():
    """A decode that scaled subnormals by 2^-25 instead of 2^-24 fails the
    binary16 pin on every nonzero subnormal."""
    want = np.arange(65536, dtype=np.uint16).view(np.float16).astype(np.float32)
    m = np.arange(1, 1024)
    bad = np.ldexp(m.astype(np.float64), -25).astype(np.float32)   # planted
    assert not np.array_equal(bad, want[1:1024])
