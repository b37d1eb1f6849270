"""Exact-arithmetic pins of the oracle's bit-exact steps (CPU, no GPU).

The quantizer's code is clamp(rint((x - mn) / scale), 0, L - 1) with IEEE
binary32 round-to-nearest-even subtraction and division and a half-to-even
rint (SemKV, Table 2 and Table 6: integer-level affine quantization with two
scalars per row).  The reference below is written from those definitions with
Python's exact rationals: every fp32 operation is the exact rational result
rounded to binary32 by an explicit nearest-even rule, and rint is an exact
comparison of the fractional part with 1/2.  It uses no floating-point
division or rounding of numpy, so a slip in the oracle's tie rule (half-up
instead of half-to-even) or in its division (a reciprocal product instead of
the IEEE quotient) fails here.

The key-norm pins are hand-computed rows whose fp32 result depends on the
association order that the key-L2 reading fixes (lane partials of four dims,
an xor butterfly over 16, 8, 4, 2, 1, heads added in index order).
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import semkv_oracle as O

HALF = Fraction(1, 2)


def rn32(q: Fraction) -> float:
    """Exact rational -> nearest binary32 value, ties to the even significand
    (normal and subnormal range; the values here never overflow)."""
    q = Fraction(q)
    if q == 0:
        return 0.0
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)                       # below 2^-126 the quantum stays 2^-149
    quantum = Fraction(2) ** (e - 23)
    m = a / quantum
    n = m.numerator // m.denominator
    r = m - n
    if r > HALF or (r == HALF and n % 2 == 1):
        n += 1
    return sign * float(n * quantum)      # exact: n * quantum is a binary32 value


def rint_half_even(t: Fraction) -> int:
    t = Fraction(t)
    f = math.floor(t)
    r = t - f
    if r > HALF or (r == HALF and f % 2 == 1):
        return f + 1
    return f


def exact_quantize_row(x16: np.ndarray, L: int):
    """Codes, mn, scale of one fp16 row by the definition, in exact rationals."""
    xs = [Fraction(float(v)) for v in x16.astype(np.float32)]
    mn, mx = min(xs), max(xs)                       # +0 canonicalisation does not change a rational
    scale = Fraction(rn32(Fraction(rn32(mx - mn)) / (L - 1)))
    codes = []
    for x in xs:
        if scale == 0:
            codes.append(0)
            continue
        d = Fraction(rn32(x - mn))
        t = Fraction(rn32(d / scale))
        codes.append(min(max(rint_half_even(t), 0), L - 1))
    return np.array(codes, dtype=np.uint8), float(mn), float(scale)


def test_rn32_matches_known_roundings():
    # the rounding helper itself, on values whose binary32 rounding is known
    assert rn32(Fraction(1, 3)) == float(np.float32(1 / 3))
    assert rn32(Fraction(1) + Fraction(1, 2 ** 24)) == 1.0                    # tie -> even (1.0)
    assert rn32(Fraction(1) + Fraction(3, 2 ** 24)) == 1.0 + 2.0 ** -22       # tie -> even (...10)
    assert rn32(Fraction(1) + Fraction(1, 2 ** 24) + Fraction(1, 2 ** 60)) == 1.0 + 2.0 ** -23
    assert rn32(Fraction(-5, 7)) == -float(np.float32(5 / 7))
    assert rn32(Fraction(1, 2 ** 149)) == 2.0 ** -149                         # smallest subnormal
    assert rint_half_even(Fraction(5, 2)) == 2 and rint_half_even(Fraction(7, 2)) == 4
    assert rint_half_even(Fraction(-1, 2)) == 0 and rint_half_even(Fraction(51, 100)) == 1


def test_quantize_exact_half_integers_round_to_even():
    # L = 6, min 0, max 5: scale = 1 exactly and every t = x is exact, so the
    # halves 0.5, 1.5, ..., 4.5 are true ties: half-to-even gives 0, 2, 2, 4, 4
    L = 6
    vals = [0.0, 5.0, 0.5, 1.5, 2.5, 3.5, 4.5]
    x = np.zeros(128, dtype=np.float16)
    x[: len(vals)] = vals
    c, mn, sc, bad = O.quantize_rows(x[None], L)
    assert not bad[0] and mn[0] == 0 and sc[0] == 1
    assert c[0, : len(vals)].tolist() == [0, 5, 0, 2, 2, 4, 4]
    ref, _, _ = exact_quantize_row(x, L)
    assert np.array_equal(c[0], ref)
    # the same ties under a non-unit scale: min -3, max 7, L = 5 -> scale 2.5,
    # x = -3 + (k + 1/2) * 2.5 for k = 0..3
    L = 5
    x = np.full(128, -3.0, dtype=np.float16)
    x[1] = 7.0
    x[2:6] = [-3 + (k + 0.5) * 2.5 for k in range(4)]
    c, mn, sc, _ = O.quantize_rows(x[None], L)
    assert sc[0] == np.float32(2.5)
    assert c[0, 2:6].tolist() == [0, 2, 2, 4]
    assert np.array_equal(c[0], exact_quantize_row(x, L)[0])


def _division_flip_cases(levels=(5, 6), n_max=160):
    """(L, mx, x) with min 0 where rint(RN(x / scale)) and
    rint(RN(x * RN(1 / scale))) differ: x is an fp16 value next to
    (k + 1/2) * scale.  Found by exact rational search, never by a kernel."""
    out = []
    mxs = np.arange(0x3C00, 0x4C00, 7, dtype=np.uint16).view(np.float16)[:n_max]   # [1, 32)
    for L in levels:
        for mx in mxs:
            mxf = Fraction(float(mx))
            scale = Fraction(rn32(mxf / (L - 1)))
            rcp = Fraction(rn32(1 / scale))
            for k in range(L - 1):
                c16 = np.float16((k + 0.5) * float(scale))
                for cand in (np.nextafter(c16, np.float16(-1)), c16, np.nextafter(c16, np.float16(100))):
                    d = Fraction(float(cand))
                    if d < 0 or d > mxf:
                        continue
                    c_div = rint_half_even(Fraction(rn32(d / scale)))
                    c_rcp = rint_half_even(Fraction(rn32(d * rcp)))
                    if min(c_div, L - 1) != min(c_rcp, L - 1):
                        out.append((L, float(mx), float(cand), min(c_div, L - 1)))
    return out


def test_quantize_uses_ieee_division_not_reciprocal_product():
    cases = _division_flip_cases()
    assert len(cases) >= 20                  # the search finds such rows in quantity
    rows, want = [], []
    for L, mx, x, code in cases:
        r = np.zeros(128, dtype=np.float16)
        r[1], r[2] = mx, x                   # min 0 (dim 0), max mx, the flip value
        rows.append((L, r))
        want.append(code)
    for L in sorted({L for L, _ in rows}):
        idx = [i for i, (LL, _) in enumerate(rows) if LL == L]
        x = np.stack([rows[i][1] for i in idx])
        c, _, _, bad = O.quantize_rows(x, L)
        assert not bad.any()
        assert c[:, 2].tolist() == [want[i] for i in idx]


@pytest.mark.parametrize("L", [2, 3, 5, 6, 7, 11, 16])
def test_quantize_matches_exact_rational_definition(L):
    # random rows plus rows with several values on or next to half-integer codes
    rng = np.random.default_rng(500 + L)
    x = (rng.standard_normal((24, 128)) * rng.lognormal(0, 1, (24, 1))).astype(np.float16)
    grid = np.zeros((8, 128), dtype=np.float16)
    for i in range(8):
        mn, step = float(np.float16(-1 - i)), float(np.float16(0.5 + 0.25 * i))
        kk = rng.integers(0, 2 * (L - 1) + 1, 128) / 2.0          # halves of the step
        kk[0], kk[1] = 0, L - 1
        grid[i] = (mn + kk * step).astype(np.float16)
    x = np.concatenate([x, grid])
    c, mn, sc, bad = O.quantize_rows(x, L)
    assert not bad.any()
    for i in range(x.shape[0]):
        ref, rmn, rsc = exact_quantize_row(x[i], L)
        assert mn[i] == np.float32(rmn) and sc[i] == np.float32(rsc)
        assert np.array_equal(c[i], ref), (L, i, np.nonzero(c[i] != ref))


# ---------------------------------------------------------------- key-L2 order
def test_key_l2_butterfly_order_hand_computed():
    # One head.  Dim 0 = 1 (lane 0); dims 4, 12, 20, 28 = 2^-12 (lanes 1, 3, 5, 7,
    # squares 2^-24 each).  In the fixed order lane 0 meets the odd lanes only at
    # the last butterfly step (xor 1), after the four 2^-24 have been summed
    # exactly among the odd lanes: acc = 1 + 2^-22, sqrt = 1 + 2^-23.  Adding
    # them to 1 one at a time (xor 1 first, or plain dim order) loses each one
    # to the tie-to-even rule and gives exactly 1.
    k = np.zeros((1, 1, 128), dtype=np.float16)
    k[0, 0, 0] = 1.0
    for d in (4, 12, 20, 28):
        k[0, 0, d] = np.float16(2.0 ** -12)
    s = O.score_key_l2(k)
    assert s[0] == np.float32(1.0 + 2.0 ** -23)


def test_key_l2_head_order_hand_computed():
    # Four heads, one nonzero per head: head 0 holds 1, heads 1..3 hold 2^-12
    # (squares 2^-24).  Heads are added in index order starting from 0:
    # ((1 + 2^-24) + 2^-24) + 2^-24, each addition a tie that rounds back to 1,
    # so the score is exactly 1.  Summing heads 3, 2, 1 first would give
    # 1 + 3*2^-24 -> 1 + 2^-22 and a score of 1 + 2^-23.
    k = np.zeros((4, 1, 128), dtype=np.float16)
    k[0, 0, 0] = 1.0
    k[1:, 0, 0] = np.float16(2.0 ** -12)
    assert O.score_key_l2(k)[0] == np.float32(1.0)
    # two heads: the per-head totals (1 and 4 * 2^-24 from the odd lanes) meet
    # only in the head sum: 1 + 2^-22 exactly, sqrt = 1 + 2^-23
    k2 = np.zeros((2, 1, 128), dtype=np.float16)
    k2[0, 0, 0] = 1.0
    for d in (4, 12, 20, 28):
        k2[1, 0, d] = np.float16(2.0 ** -12)
    assert O.score_key_l2(k2)[0] == np.float32(1.0 + 2.0 ** -23)
