"""The scalar arithmetic of the quantize kernel, checked on the CPU.

quantize.cu computes the stored scale RN((mx - mn) / (L - 1)) without a divide:
    q0 = RN(a * rk),  r = fma(-q0, k, a),  scale = fma(r, rk, q0),
with k = L - 1 and rk = RN(1 / k) (a quotient corrected once by its exact
residual).  These tests emulate each fused multiply-add exactly in numpy and
check the result against numpy's IEEE float32 division for every significand
and every k in 1..15 (a power-of-two factor of a scales the quotient exactly,
so one binade covers all finite a).

The codes take the same correction for a general divisor: with r = RN(1/scale),
    q0 = RN(d * r),  rem = fma(-q0, scale, d),  q = fma(rem, r, q0)
is RN(d / scale) (Markstein's theorem).  The last test checks that on random
divisors and on quotients driven onto and around every half-integer below 16,
where rint decides between two codes.
"""
import numpy as np

F32 = np.float32


def _fma32(a, b, c):
    """RN32(a*b + c) exactly, for float32 arrays (no overflow)."""
    p = a.astype(np.float64) * b.astype(np.float64)        # exact: 48-bit product
    c64 = c.astype(np.float64)
    s = p + c64
    bp = s - c64                                            # TwoSum: s + err == p + c exactly
    err = (p - bp) + (c64 - (s - bp))
    r = s.astype(F32)
    # float64 -> float32 rounding is only wrong when s sits exactly on a float32
    # midpoint and err breaks the tie
    lo = np.where(r.astype(np.float64) > s, np.nextafter(r, F32(-np.inf)), r)
    hi = np.nextafter(lo, F32(np.inf))
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) * 0.5
    tie = (s == mid) & (err != 0)
    return np.where(tie, np.where(err > 0, hi, lo), r)


def test_fma_emulation_breaks_ties_by_the_exact_sum():
    one = np.array([1.0], F32)
    eps = np.array([2.0 ** -24], F32)                 # half an ulp of 1
    tiny = np.array([2.0 ** -60], F32)
    assert _fma32(tiny, one, one)[0] == F32(1.0)
    assert _fma32(eps, one, one)[0] == F32(1.0)                 # exact tie 1 + 2^-24 -> even
    a = np.array([1.0 + 2.0 ** -23], F32)
    b = np.array([1.0 + 2.0 ** -23], F32)
    # (1 + 2^-23)^2 = 1 + 2^-22 + 2^-46: exact sum above the float32 grid point
    assert _fma32(a, b, np.array([0.0], F32))[0] == F32(1.0 + 2.0 ** -22)
    # a product that lands exactly between two float32 values, nudged by c
    x = np.array([1.0 + 2.0 ** -12], F32)
    prod = x.astype(np.float64) ** 2                            # 1 + 2^-11 + 2^-24: a midpoint
    assert F32(prod) == F32(1.0 + 2.0 ** -11)                   # tie to even
    up = _fma32(x, x, np.array([2.0 ** -70], F32))[0]
    dn = _fma32(x, x, np.array([-2.0 ** -70], F32))[0]
    assert up == np.nextafter(F32(1.0 + 2.0 ** -11), F32(2)) and dn == F32(1.0 + 2.0 ** -11)


def test_corrected_product_is_the_ieee_quotient_for_every_significand():
    a = (np.arange(1 << 23, dtype=np.uint32) | np.uint32(127 << 23)).view(F32)   # all of [1, 2)
    for k in range(1, 16):
        kf = np.full(a.shape, k, F32)
        rk = np.full(a.shape, F32(1) / F32(k), F32)
        q0 = (a.astype(np.float64) * rk.astype(np.float64)).astype(F32)          # RN(a * rk)
        r = _fma32(-q0, kf, a)
        q1 = _fma32(r, rk, q0)
        ref = a / F32(k)
        bad = np.count_nonzero(q1 != ref)
        assert bad == 0, f"k={k}: {bad} significands differ from the IEEE quotient"


def test_corrected_quotient_is_the_ieee_quotient_near_every_half_integer():
    rng = np.random.default_rng(17)
    n = 1 << 21
    scale = (rng.uniform(1.0, 2.0, n) * 2.0 ** rng.integers(-28, 10, n)).astype(F32)
    # d/scale on and within a few ulps of the half-integers 0.5 .. 15.5, and anywhere in [0, 16)
    t = ((rng.integers(0, 16, n) + 0.5) * scale.astype(np.float64)).astype(F32)
    d_tie = (t.view(np.uint32).astype(np.int64) + rng.integers(-4, 5, n)).astype(np.uint32).view(F32)
    d_any = (rng.uniform(0.0, 16.0, n) * scale.astype(np.float64)).astype(F32)
    for d in (d_tie, d_any):
        r = F32(1) / scale                                           # RN(1/scale)
        q0 = (d.astype(np.float64) * r.astype(np.float64)).astype(F32)
        rem = _fma32(-q0, scale, d)
        q = _fma32(rem, r, q0)
        assert np.array_equal(q, d / scale)
        magic = np.full(n, 1.5 * 2.0 ** 23, F32)
        assert np.array_equal((q + magic) - magic, np.rint(d / scale))
