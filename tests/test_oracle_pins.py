"""Pins of the CPU oracle to things other than itself (runs on CPU, no GPU).

Each test checks the oracle against a closed form, a brute force on tiny inputs,
a textbook or library special case, or a value printed on the SemKV page
(tests/golden/), chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong tie rule) fails one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

from oracle import semkv_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- a0 num_high
def test_num_high_matches_exact_rational_ceiling():
    rng = np.random.default_rng(0)
    for _ in range(2000):
        n = int(rng.integers(0, 300_000))
        r = int(rng.integers(0, 1_000_001))
        assert O.num_high(n, r) == math.ceil(Fraction(r, 1_000_000) * n)


def test_num_high_special_values():
    assert O.num_high(32768, 100_000) == 3277          # 0.1 * 32768 = 3276.8
    assert O.num_high(128, 500_000) == 64
    assert O.num_high(128, 250_000) == 32
    assert O.num_high(77, 0) == 0
    assert O.num_high(77, 1_000_000) == 77
    assert O.num_high(0, 500_000) == 0


# ---------------------------------------------------------------- layout sizes
@pytest.mark.parametrize("L,n,W", [(2, 32, 4), (3, 20, 7), (4, 16, 8), (5, 13, 10),
                                   (6, 12, 11), (8, 10, 13), (16, 8, 16)])
def test_digits_and_words_closed_form(L, n, W):
    assert O.digits_per_word(L) == n
    assert O.digits_per_word(L) == math.floor(32 / math.log2(L))
    assert O.words_per_row(L) == W == math.ceil(128 / n)


def test_layout_code_bits_approach_log2_levels():
    # code bits per value of the layout (32 / n) exceed log2 L by less than one digit's share
    for L in range(2, 17):
        n = O.digits_per_word(L)
        assert math.log2(L) <= 32 / n < math.log2(L) * (n + 1) / n + 1e-12


# ---------------------------------------------------------------- printed storage figures
def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([c.strip() for c in line.split("|")])
    return rows


def test_printed_code_bits():
    for L, bits, _ in _golden_rows("code_bits.txt"):
        assert round(O.pages_code_bits(int(L)), 3) == float(bits)


def test_printed_effective_bits_and_compression():
    rows = _golden_rows("storage_table.txt")
    assert len(rows) == 12
    for name, mix, meta, eff, comp, _ in rows:
        lf = [(int(a), float(b)) for a, b in (p.split(":") for p in mix.split(","))]
        e = O.pages_effective_bits(lf, int(meta))
        if eff != "-":
            assert round(e, 3) == float(eff), name
        if comp != "-":
            assert round(16 / e, 1) == float(comp), name


def test_printed_nominal_bits_and_pruning_ratio():
    # Table 3: 2.39 nominal average code bits at 25% of 6 levels + 75% of 5 levels
    assert round(0.25 * math.log2(6) + 0.75 * math.log2(5), 2) == 2.39
    # Table 4 / Fig. 11: FP16 keep-25% pruning (4.0 bits) occupies 1.5x SemKV's footprint
    semkv = O.pages_effective_bits([(6, 0.25), (5, 0.75)], 2)
    assert round(16 * 0.25 / semkv, 1) == 1.5
    assert round(16 / (16 * 0.25), 1) == 4.0


# ---------------------------------------------------------------- a1' key L2
def test_key_l2_close_to_float64_norm():
    rng = np.random.default_rng(1)
    k = (rng.standard_normal((8, 300, 128)) * rng.lognormal(0, 1, (8, 1, 128))).astype(np.float16)
    s = O.score_key_l2(k)
    ref = np.sqrt((k.astype(np.float64) ** 2).sum(axis=(0, 2)))
    assert s.dtype == np.float32
    assert np.max(np.abs(s / ref - 1)) < 2 ** -20


def test_key_l2_special_cases():
    k = np.zeros((3, 5, 128), dtype=np.float16)
    k[1, 2, 77] = np.float16(-3.5)      # one nonzero entry: sqrt(x^2) == |x| exactly
    k[2, 4, 0] = np.float16(6.0)
    k[0, 4, 127] = np.float16(8.0)      # 6-8-10 triangle across heads
    s = O.score_key_l2(k)
    assert s[0] == 0 and s[1] == 0 and s[3] == 0
    assert s[2] == np.float32(3.5)
    assert s[4] == np.float32(10.0)
    # power-of-two scaling commutes with every rounding step
    rng = np.random.default_rng(2)
    k = rng.standard_normal((2, 50, 128)).astype(np.float16)
    assert np.array_equal(O.score_key_l2((k * np.float16(4)).astype(np.float16)), 4 * O.score_key_l2(k))


# ---------------------------------------------------------------- a1 attention mass
def test_attn_mass_total_is_number_of_rows():
    rng = np.random.default_rng(3)
    H, H_q, T, w = 2, 8, 97, 16
    k = rng.standard_normal((H, T, 128)).astype(np.float16)
    q = rng.standard_normal((H_q, w, 128)).astype(np.float16)
    s = O.score_attn_mass(k, q, T)
    assert abs(s.sum() - H_q * w) < 1e-9
    # causal: the last key is seen only by the last window row of each head
    assert np.all(s >= 0)


def test_attn_mass_equal_keys_closed_form():
    H, H_q, T, w = 1, 4, 50, 8
    k = np.ones((H, T, 128), dtype=np.float16)
    q = np.random.default_rng(4).standard_normal((H_q, w, 128)).astype(np.float16)
    s = O.score_attn_mass(k, q, T)
    pos = T - w + np.arange(w)
    expect = np.array([H_q * sum(1.0 / (p + 1) for p in pos if p >= j) for j in range(T)])
    assert np.allclose(s, expect, rtol=1e-12, atol=1e-12)


def test_attn_mass_single_row_is_scipy_softmax():
    rng = np.random.default_rng(5)
    T = 64
    k = rng.standard_normal((1, T, 128)).astype(np.float16)
    q = rng.standard_normal((1, 1, 128)).astype(np.float16)
    s = O.score_attn_mass(k, q, T)
    ref = scipy.special.softmax(k[0].astype(np.float64) @ q[0, 0].astype(np.float64) / math.sqrt(128))
    assert np.allclose(s, ref, rtol=1e-12, atol=1e-15)


def test_attn_mass_gqa_head_mapping():
    # H=2 KV heads, H_q=4: query heads 0,1 read KV head 0; heads 2,3 read KV head 1.
    rng = np.random.default_rng(6)
    T = 40
    k = np.zeros((2, T, 128), dtype=np.float16)
    k[0] = rng.standard_normal((T, 128)).astype(np.float16)      # KV head 1 all zero
    q = rng.standard_normal((4, 1, 128)).astype(np.float16)
    s = O.score_attn_mass(k, q, T)
    ref = np.zeros(T)
    for h in (0, 1):
        ref += scipy.special.softmax(k[0].astype(np.float64) @ q[h, 0].astype(np.float64) / math.sqrt(128))
    ref += 2.0 / T                                                # heads 2, 3: uniform
    assert np.allclose(s, ref, rtol=1e-12, atol=1e-15)


def test_attn_mass_short_sequence_skips_rows():
    rng = np.random.default_rng(7)
    T, w = 5, 8
    k = rng.standard_normal((1, T, 128)).astype(np.float16)
    q = rng.standard_normal((4, w, 128)).astype(np.float16)
    s = O.score_attn_mass(k, q, T)
    assert abs(s.sum() - 4 * T) < 1e-9     # only the T rows with position >= 0 count


# ---------------------------------------------------------------- a2 select
def test_select_brute_force_with_ties():
    rng = np.random.default_rng(8)
    for trial in range(300):
        T = int(rng.integers(1, 40))
        pool = np.array([0.0, -0.0, 1.5, 1.5, -2.0, 3.25, 1e-30, -1e-30], dtype=np.float32)
        s = rng.choice(pool, T) if trial % 2 else rng.standard_normal(T).astype(np.float32)
        n_high = int(rng.integers(0, T + 1))
        mask = O.select_mask(s, n_high)
        ranked = sorted(range(T), key=lambda j: (-float(s[j]) if s[j] != 0 else 0.0, j))
        expect = np.zeros(T, dtype=np.uint8)
        expect[ranked[:n_high]] = 1
        assert np.array_equal(mask, expect)
        assert int(mask.sum()) == n_high and int((1 - mask).sum()) == T - n_high


def test_select_ties_go_to_lower_index():
    s = np.array([1, 2, 2, 2, 0, 2], dtype=np.float32)
    assert O.select_mask(s, 2).tolist() == [0, 1, 1, 0, 0, 0]
    assert O.select_mask(np.array([0.0, -0.0, 0.0], np.float32), 1).tolist() == [1, 0, 0]
    assert O.select_mask(np.array([-0.0, 0.0], np.float32), 1).tolist() == [1, 0]


# ---------------------------------------------------------------- a3/a4 quantize
def _rows(rng, R, scale=1.0):
    x = rng.standard_normal((R, 128)) * scale
    return x.astype(np.float16)


@pytest.mark.parametrize("L", list(range(2, 17)))
def test_quantize_codes_range_extremes_and_error_bound(L):
    rng = np.random.default_rng(100 + L)
    x = np.concatenate([_rows(rng, 200), _rows(rng, 50, 1000.0), _rows(rng, 50, 1e-3)])
    c, mn, sc, bad = O.quantize_rows(x, L)
    assert not bad.any()
    assert c.max() <= L - 1
    xf = x.astype(np.float32)
    r = np.arange(x.shape[0])
    assert np.all(c[r, xf.argmin(1)] == 0)
    assert np.all(c[r, xf.argmax(1)] == L - 1)
    xhat = O.dequantize(c, mn, sc)
    err = np.abs(xf.astype(np.float64) - xhat)
    bound = sc[:, None] * (0.5 + 2 ** -20) + 2 ** -22 * np.maximum(np.abs(mn), np.abs(xf.max(1)))[:, None]
    assert np.all(err <= bound)
    # monotone in x within a row
    order = np.argsort(xf, axis=1, kind="stable")
    assert np.all(np.diff(np.take_along_axis(c.astype(int), order, 1), axis=1) >= 0)


def test_quantize_exact_grid_rows():
    rng = np.random.default_rng(9)
    for L in (3, 5, 6, 8, 16):
        k = rng.integers(0, L, 128)
        k[0], k[1] = 0, L - 1
        mn, step = -2.0, 0.25
        x = (mn + k * step).astype(np.float16)
        c, m, s, _ = O.quantize_rows(x[None], L)
        assert m[0] == np.float32(mn) and s[0] == np.float32(step * (L - 1) / (L - 1))
        assert np.array_equal(c[0], k.astype(np.uint8))


def test_quantize_constant_rows_and_signed_zero():
    x = np.full((3, 128), 0.0, dtype=np.float16)
    x[1] = np.float16(-0.0)
    x[2] = np.float16(7.25)
    c, mn, sc, bad = O.quantize_rows(x, 6)
    assert not bad.any() and np.all(c == 0) and np.all(sc == 0)
    assert np.signbit(mn).sum() == 0            # -0 canonicalised to +0
    assert mn[2] == np.float32(7.25)


def test_quantize_nonfinite_rows_flagged():
    x = np.zeros((3, 128), dtype=np.float16)
    x[0, 5] = np.float16(np.inf)
    x[2, 9] = np.float16(np.nan)
    _, _, _, bad = O.quantize_rows(x, 5)
    assert bad.tolist() == [True, False, True]


@pytest.mark.parametrize("L", [2, 3, 4, 5, 6, 8, 16])
def test_quantize_uniform_case_matches_textbook_minmax(L):
    # textbook per-token min-max quantization in float64; float32 may differ only
    # where (x - min) / scale lies within a hair of a half-integer
    rng = np.random.default_rng(200 + L)
    x = _rows(rng, 500)
    c, _, _, _ = O.quantize_rows(x, L)
    xd = x.astype(np.float64)
    lo, hi = xd.min(1, keepdims=True), xd.max(1, keepdims=True)
    t = (xd - lo) / ((hi - lo) / (L - 1))
    ref = np.clip(np.floor(t + 0.5), 0, L - 1)
    diff = c != ref
    near_half = np.abs(t - np.floor(t) - 0.5) < 1e-5
    assert np.all(~diff | near_half)
    assert diff.mean() < 1e-3


# ---------------------------------------------------------------- pack
@pytest.mark.parametrize("L", list(range(2, 17)))
def test_pack_roundtrip_and_word_range(L):
    rng = np.random.default_rng(300 + L)
    c = rng.integers(0, L, (64, 128)).astype(np.uint8)
    c[0] = L - 1
    w = O.pack_rows(c, L)
    assert w.dtype == np.uint32 and w.shape == (64, O.words_per_row(L))
    assert np.array_equal(O.unpack_rows(w, L), c)
    n = O.digits_per_word(L)
    # first word of the all-max row: L**n - 1 (fits in 32 bits by construction)
    assert int(w[0, 0]) == L ** n - 1


@pytest.mark.parametrize("L,bits", [(2, 1), (4, 2), (16, 4)])
def test_pack_equals_bit_packing_for_powers_of_two(L, bits):
    rng = np.random.default_rng(400 + L)
    c = rng.integers(0, L, (32, 128)).astype(np.uint8)
    w = O.pack_rows(c, L)
    per = 32 // bits
    for r in range(32):
        for wi in range(w.shape[1]):
            acc = 0
            for j in range(per):
                acc |= int(c[r, wi * per + j]) << (bits * j)
            assert int(w[r, wi]) == acc


def test_pack_digit_order_little_endian():
    c = np.zeros((1, 128), np.uint8)
    c[0, 1] = 1                      # second digit of the first word
    c[0, 12] = 2                     # first digit of the second word (L=6, n=12)
    w = O.pack_rows(c, 6)
    assert int(w[0, 0]) == 6 and int(w[0, 1]) == 2 and int(w[0, 2:].sum()) == 0


# ---------------------------------------------------------------- pools and generation
def test_slab_pools_keep_token_order_and_every_token():
    rng = np.random.default_rng(10)
    x = _rows(rng, 70)
    mask = O.select_mask(rng.random(70).astype(np.float32), O.num_high(70, 250_000))
    ph, pl, _ = O.quantize_slab(x, mask, 6, 5)
    assert ph.words.shape[0] == 18 and pl.words.shape[0] == 52
    hi_tok = np.nonzero(mask)[0]
    ch, mh, sh, _ = O.quantize_rows(x[hi_tok[3:4]], 6)
    assert np.array_equal(ph.words[3], O.pack_rows(ch, 6)[0]) and ph.mn[3] == mh[0]


def test_generation_block_exact_counts():
    rng = np.random.default_rng(11)
    B, Lyr, H = 2, 1, 1
    cache = O.MixedCache(B, Lyr, H, 6, 5, 500_000, block=16)
    T = 20
    k = rng.standard_normal((B, Lyr, H, T, 128)).astype(np.float16)
    masks = [O.select_mask(rng.random(T).astype(np.float32), O.num_high(T, 500_000)) for _ in range(B)]
    cache.prefill(k, k, [T, T], masks)
    assert cache.n_high.tolist() == [10, 10]
    total = T
    for step in range(40):
        kn = rng.standard_normal((B, Lyr, H, 1, 128)).astype(np.float16)
        cache.append(kn, kn, rng.random((B, 1)).astype(np.float32))
        total += 1
        assert cache.buf_k.shape[3] < 16                    # a full block never stays FP16
        blocks = (total - T) // 16
        assert cache.n_high.tolist() == [10 + 8 * blocks] * B
        assert (cache.n_high + cache.n_low + cache.buf_k.shape[3]).tolist() == [total] * B
    res = cache.buf_k.shape[3]                                # 40 = 2*16 + 8
    assert res == 8
    cache.flush()
    assert cache.n_high.tolist() == [10 + 16 + O.num_high(8, 500_000)] * B
    assert cache.buf_k.shape[3] == 0


# ---------------------------------------------------------------- rotation (Hadamard, Table 2)
def test_fwht128_matches_scipy_hadamard_matrix():
    import scipy.linalg
    Hm = scipy.linalg.hadamard(128).astype(np.float64)
    rng = np.random.default_rng(31)
    xi = rng.integers(-50, 51, (20, 128)).astype(np.float64)        # exact in any order
    assert np.array_equal(O.fwht128(xi), xi @ Hm.T)
    assert np.array_equal(O.fwht128(O.fwht128(xi)), 128.0 * xi)       # H H = 128 I
    x = (rng.standard_normal((50, 128)) * rng.lognormal(0, 2, (50, 1))).astype(np.float32)
    y = O.fwht128(x)
    assert y.dtype == np.float32
    exact = x.astype(np.float64) @ Hm.T
    bound = 7 * 2.0 ** -24 * np.abs(x.astype(np.float64)).sum(axis=1, keepdims=True) * 2
    assert np.all(np.abs(y - exact) <= bound)


def test_rotated_quantizer_error_bound_and_outlier_spread():
    # x_hat = H(dequant(q(Hx)))/128: each rotated value errs by at most
    # scale/2 (+ fp32 slack), and the inverse transform averages 128 of them
    rng = np.random.default_rng(32)
    T = 400
    x = rng.standard_normal((T, 128)).astype(np.float32)
    x[:, [3, 50, 77, 120]] *= 10.0                                    # four outlier channels
    xh = x.astype(np.float16)
    for L in (5, 6):
        mask = np.zeros(T, np.uint8) if L == 5 else np.ones(T, np.uint8)
        ph, pl, bad = O.quantize_slab(xh, mask, 6, 5, rotate=True)
        pool = ph if L == 6 else pl
        rec = O.fwht128(O.dequantize(O.unpack_rows(pool.words, L), pool.mn, pool.scale)) / 128.0
        err = np.abs(rec - xh.astype(np.float64))
        assert not bad.any()
        assert np.all(err <= pool.scale[:, None] * (0.5 + 2.0 ** -18) + 1e-5 * np.abs(pool.mn)[:, None] + 1e-6)
        # outliers: the rotation spreads the four large channels over every dim,
        # so the mean squared error is lower than without it
        p2h, p2l, _ = O.quantize_slab(xh, mask, 6, 5, rotate=False)
        p2 = p2h if L == 6 else p2l
        rec2 = O.dequantize(O.unpack_rows(p2.words, L), p2.mn, p2.scale)
        assert np.mean(err ** 2) < 0.5 * np.mean((rec2 - xh.astype(np.float64)) ** 2)


# ---------------------------------------------------------------- a6 decode
def test_decode_all_fp16_buffer_is_textbook_attention():
    rng = np.random.default_rng(12)
    B, Lyr, H, H_q = 1, 2, 2, 8
    cache = O.MixedCache(B, Lyr, H, 6, 5, 500_000)
    kn = rng.standard_normal((B, Lyr, H, 50, 128)).astype(np.float16)
    vn = rng.standard_normal((B, Lyr, H, 50, 128)).astype(np.float16)
    cache.append(kn, vn, rng.random((B, 50)).astype(np.float32))
    q = rng.standard_normal((B, Lyr, H_q, 128)).astype(np.float16)
    out = cache.decode(q)
    qt = torch.from_numpy(q.astype(np.float64)).reshape(B * Lyr, H_q, 1, 128)
    kt = torch.from_numpy(kn.astype(np.float64)).reshape(B * Lyr, H, 50, 128)
    vt = torch.from_numpy(vn.astype(np.float64)).reshape(B * Lyr, H, 50, 128)
    kt = kt.repeat_interleave(H_q // H, dim=1)
    vt = vt.repeat_interleave(H_q // H, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).reshape(B, Lyr, H_q, 128)
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_buffer_mass_all_fp16_cache_sums_to_query_heads_and_matches_scipy():
    # every key in the FP16 block: each head's probabilities sum to 1, and the
    # mass equals scipy's softmax summed over the heads of each KV head
    rng = np.random.default_rng(21)
    B, Lyr, H, H_q, n = 2, 2, 2, 8, 37
    cache = O.MixedCache(B, Lyr, H, 6, 5, 500_000)
    kn = rng.standard_normal((B, Lyr, H, n, 128)).astype(np.float16)
    cache.append(kn, kn, np.zeros((B, n), np.float32))
    q = rng.standard_normal((B, Lyr, H_q, 128)).astype(np.float16)
    cache.decode(q, score_layer=1)
    for b in range(B):
        assert abs(float(cache.buf_score[b].astype(np.float64).sum()) - H_q) < 1e-4
        ref = np.zeros(n)
        for h in range(H_q):
            lg = kn[b, 1, h // (H_q // H)].astype(np.float64) @ q[b, 1, h].astype(np.float64) / math.sqrt(128)
            ref += scipy.special.softmax(lg)
        assert np.allclose(cache.buf_score[b], ref, rtol=1e-6, atol=1e-7)
    # a second step accumulates; a step at another layer adds nothing
    before = cache.buf_score.copy()
    cache.decode(q, score_layer=1)
    assert np.allclose(cache.buf_score, 2 * before.astype(np.float64), rtol=1e-6)
    cache.decode(q, score_layer=None)
    cache.decode(q[:, :1], layer0=0, score_layer=1)            # layer 1 not decoded: no change
    assert np.allclose(cache.buf_score, 2 * before.astype(np.float64), rtol=1e-6)


def test_buffer_mass_equal_keys_is_uniform_over_pools_and_block():
    # identical keys everywhere (a constant row quantizes losslessly): every
    # cached token gets 1/n of each head, so a block token gets H_q / n
    B, Lyr, H, H_q, T, nb = 1, 1, 1, 4, 30, 5
    cache = O.MixedCache(B, Lyr, H, 6, 5, 500_000)
    k = np.full((B, Lyr, H, T, 128), 0.75, np.float16)
    cache.prefill(k, k, [T], [O.select_mask(np.arange(T, dtype=np.float32), O.num_high(T, 500_000))])
    kb = np.full((B, Lyr, H, nb, 128), 0.75, np.float16)
    cache.append(kb, kb, np.zeros((B, nb), np.float32))
    q = np.random.default_rng(3).standard_normal((B, Lyr, H_q, 128)).astype(np.float16)
    cache.decode(q, score_layer=0)
    assert np.allclose(cache.buf_score[0], H_q / (T + nb), rtol=1e-6)


def test_decode_lossless_grid_cache_is_textbook_attention():
    # rows built on their own class's level grid quantize without loss, so the
    # mixed-cache decode must equal plain attention over the same values
    rng = np.random.default_rng(13)
    B, Lyr, H, H_q, T = 2, 2, 2, 8, 90
    masks = [O.select_mask(rng.random(T).astype(np.float32), O.num_high(T, 250_000)) for _ in range(B)]

    def grid_rows():
        x = np.zeros((B, Lyr, H, T, 128))
        for b in range(B):
            for t in range(T):
                L = 6 if masks[b][t] else 5
                k = rng.integers(0, L, (Lyr, H, 128))
                k[..., 0], k[..., 1] = 0, L - 1
                x[b, :, :, t] = rng.choice([-2.0, 0.5, 3.0]) + 0.25 * k
        return x.astype(np.float16)

    k, v = grid_rows(), grid_rows()
    cache = O.MixedCache(B, Lyr, H, 6, 5, 250_000)
    cache.prefill(k, v, [T] * B, masks)
    kn = rng.standard_normal((B, Lyr, H, 7, 128)).astype(np.float16)
    cache.append(kn, kn, rng.random((B, 7)).astype(np.float32))
    q = rng.standard_normal((B, Lyr, H_q, 128)).astype(np.float16)
    out = cache.decode(q)
    kk = np.concatenate([k, kn], axis=3).astype(np.float64)
    vv = np.concatenate([v, kn], axis=3).astype(np.float64)
    qt = torch.from_numpy(q.astype(np.float64)).reshape(B * Lyr, H_q, 1, 128)
    kt = torch.from_numpy(kk).reshape(B * Lyr, H, T + 7, 128).repeat_interleave(H_q // H, dim=1)
    vt = torch.from_numpy(vv).reshape(B * Lyr, H, T + 7, 128).repeat_interleave(H_q // H, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).reshape(B, Lyr, H_q, 128)
    assert np.allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)
