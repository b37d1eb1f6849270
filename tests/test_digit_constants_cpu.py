"""The f16 digit-extraction constants of the decode kernel, checked exhaustively (CPU).

decode.cu peels base-L digits off a part P of a packed word with
    t = fma(X, c, K),  X = 1024 + P (first step) or 1536 + P (later steps),
and relies on t == 1536 + floor(P / L) exactly for every part value the word
layout can produce.  This test reads the (c, K) table from the kernel source
and checks that property for every P, emulating the fused f16 multiply-add
exactly: X, c and K are f16 values, so X*c + K is exact in float64 and one
round-to-nearest-even to f16 is what the fused instruction does.  It also
checks that the part sizes cover each word and that every part stays below
1024, the range in which 1024 + P is an exact f16 integer.
"""
import os
import re

import numpy as np
import pytest

from oracle import semkv_oracle as O

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "kv_cache_mixed_b200", "csrc", "decode.cu")


def _plans():
    text = open(SRC).read()
    rows = re.findall(r"L == (\d+)\s*\?\s*F16Plan\{(\d+), \{([\d, ]+)\}, (0x[0-9a-f]+), (0x[0-9a-f]+), "
                      r"(0x[0-9a-f]+), (0x[0-9a-f]+)\}", text)
    out = {}
    for L, np_, parts, c0, k0, c1, k1 in rows:
        p = [int(x) for x in parts.split(",")][:int(np_)]
        out[int(L)] = (p, [int(v, 16) for v in (c0, k0, c1, k1)])
    return out


def _f16(bits):
    return float(np.array([bits], dtype=np.uint16).view(np.float16)[0])


def _step_ok(L, bias, pmax, c_bits, k_bits):
    P = np.arange(pmax, dtype=np.float64)
    exact = (bias + P) * _f16(c_bits) + _f16(k_bits)        # exact in float64 at these sizes
    t = exact.astype(np.float16).astype(np.float64)         # one round-to-nearest-even to f16
    return np.array_equal(t, 1536 + np.floor(P / L))


def test_every_non_power_of_two_level_has_a_plan():
    plans = _plans()
    assert sorted(plans) == [L for L in range(3, 16) if L not in (4, 8)]


@pytest.mark.parametrize("L", [L for L in range(3, 16) if L not in (4, 8)])
def test_f16_steps_are_exact_for_every_part_value(L):
    parts, (c0, k0, c1, k1) = _plans()[L]
    assert sum(parts) == O.digits_per_word(L)            # the parts cover the word's digits
    kmax = max(parts)
    assert L ** kmax <= 1024                             # 1024 + P is an exact f16 integer
    assert _step_ok(L, 1024, L ** kmax, c0, k0)          # first step of every register
    if kmax > 1:
        assert _step_ok(L, 1536, L ** (kmax - 1), c1, k1)   # every later step
    # the quotient of a pair register by multiply-high is exact: L^ka * L^(ka+kb) < 2^32
    for j in range(0, len(parts), 2):
        ka = parts[j]
        kb = parts[j + 1] if j + 1 < len(parts) else 0
        assert L ** ka * L ** (ka + kb) < 2 ** 32


@pytest.mark.parametrize("L", [L for L in range(3, 16) if L not in (4, 8)])
def test_digit_chain_reproduces_base_L_digits(L):
    """The whole f16 chain on one part, emulated step by step, gives the digits."""
    parts, (c0, k0, c1, k1) = _plans()[L]
    k = max(parts)
    P = np.arange(L ** k, dtype=np.float64)
    X = 1024 + P
    c, K, bias = _f16(c0), _f16(k0), 1024.0
    digits = []
    for s in range(k - 1):
        t = (X * c + K).astype(np.float16).astype(np.float64)
        sp = (t * -L + (1536 * L - bias)).astype(np.float16).astype(np.float64)
        digits.append((X + sp).astype(np.float16).astype(np.float64))
        X, c, K, bias = t, _f16(c1), _f16(k1), 1536.0
    digits.append((X - 1536.0 if k > 1 else X - 1024.0))
    ref = [(np.arange(L ** k) // L ** s) % L for s in range(k)]
    for s in range(k):
        assert np.array_equal(digits[s], ref[s]), (L, s)


@pytest.mark.parametrize("L", [L for L in range(3, 16) if L not in (4, 8)])
def test_floor_chain_gives_every_floor_from_its_low_bits(L):
    """The key side feeds the floors x_s = floor(P / L^s) of each part: x_0 is the
    part's raw 16-bit field, and x_s (s >= 1) is the low 9 bits of the chain's t,
    whose f16 pattern must be 0x6600 + x_s (t = 1536 + x_s with x_s < 512).  The
    floors then give the digits as d_s = x_s - L x_(s+1) (x_k = 0)."""
    parts, (c0, k0, c1, k1) = _plans()[L]
    k = max(parts)
    P = np.arange(L ** k, dtype=np.float64)
    X = 1024 + P
    c, K = _f16(c0), _f16(k0)
    floors = [P.astype(np.int64)]
    for s in range(1, k):
        t = (X * c + K).astype(np.float16)
        bits = t.view(np.uint16).astype(np.int64)
        assert np.all((bits & 0xFE00) == 0x6600), (L, s)
        floors.append(bits & 0x1FF)
        X, c, K = t.astype(np.float64), _f16(c1), _f16(k1)
    ints = np.arange(L ** k)
    for s in range(k):
        assert np.array_equal(floors[s], ints // L ** s), (L, s)
    nxt = floors[1:] + [np.zeros_like(ints)]
    for s in range(k):
        assert np.array_equal(floors[s] - L * nxt[s], (ints // L ** s) % L), (L, s)


def test_floor_coefficients_recover_the_digit_dot_product():
    """sum_s q_s d_s over a part equals q_0 x_0 + sum_(s>=1) (q_s - L q_(s-1)) x_s:
    the coefficients the key side's q fragments carry, checked on random parts."""
    rng = np.random.default_rng(7)
    for L, k in ((6, 3), (5, 4), (3, 5), (10, 3), (13, 2)):
        q = rng.standard_normal(k)
        coef = np.array([q[0]] + [q[s] - L * q[s - 1] for s in range(1, k)])
        P = rng.integers(0, L ** k, 1000)
        d = np.stack([(P // L ** s) % L for s in range(k)], 1)
        x = np.stack([P // L ** s for s in range(k)], 1)
        assert np.allclose(d @ q, x @ coef, rtol=0, atol=1e-9)


def _fp64_floor_div(x, D):
    """decode.cu div_fp64<D>: x as an exact double, inv = RN(RN(1/D) * RN(1 + 2^-50)) (IEEE double, as
    the constant is folded), then fma(x, inv, 2^52) rounded toward zero; the low word is floor(x * inv)."""
    from fractions import Fraction
    inv = (1.0 / D) * (1.0 + 2.0 ** -50)
    return int(Fraction(x) * Fraction(inv)) , inv


@pytest.mark.parametrize("L", [L for L in range(3, 16) if L not in (4, 8)])
def test_fp64_word_split_is_floor_division(L):
    # the word's first split divides by L^(p0 + p1), p0 and p1 the first two parts of the plan
    from fractions import Fraction
    parts, _ = _plans()[L]
    n = O.digits_per_word(L)
    divisors = {L ** (parts[2 * j] + parts[2 * j + 1]) for j in range((len(parts) - 1) // 2)} | \
               {L ** k for k in range(1, n + 1) if L ** k < 2 ** 32}
    rng = np.random.default_rng(L)
    for D in sorted(divisors):
        _, inv = _fp64_floor_div(0, D)
        # inv bounds 1/D from above, closely enough that x * inv never reaches the next integer
        assert Fraction(inv) >= Fraction(1, D)
        assert (2 ** 32) * (Fraction(inv) - Fraction(1, D)) * D < 1
        xs = [0, 1, D - 1, D, L ** n - 1, 2 ** 32 - 1] + [m * D + e for m in (1, 7, (2 ** 32 - 1) // D)
                                                        for e in (-1, 0, 1) if 0 <= m * D + e < 2 ** 32]
        xs += [int(v) for v in rng.integers(0, 2 ** 32, 200)]
        for x in xs:
            assert _fp64_floor_div(x, D)[0] == x // D, (L, D, x)
