"""Pins of the oracle's model of the pages' own storage layout (CPU, no GPU).

SemKV, Table 3, Table 5, Table 6 and Fig. 11 print effective bits and
compressions that "include packing and per-row metadata": groups of at most
five base-L digits in whole bits, and two 16-bit scalars per row.  The oracle
builds that layout as real bytes (pack_rows_pages: rows back to back in one bit
stream, fp16 min and scale).  These tests tie it to things other than itself:
the group choice and row sizes counted by hand, a brute-force bit reader on
tiny inputs, round trips, and the printed compressions recomputed from the
stored byte counts (tests/golden/storage_table.txt).
"""
import math
import os

import numpy as np
import pytest

from oracle import semkv_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_group_choice_matches_hand_counts():
    # 5 levels: 3 digits in 7 bits (125 <= 128); 6 levels: 5 digits in 13 bits
    # (7776 <= 8192); 8 levels: 3 bits per digit; 4 levels: 2 bits per digit
    assert O.pages_group(5) == (3, 7)
    assert O.pages_group(6) == (5, 13)
    assert O.pages_group(8)[1] / O.pages_group(8)[0] == 3
    assert O.pages_group(4)[1] / O.pages_group(4)[0] == 2
    for L in range(2, 17):
        g, b = O.pages_group(L)
        assert 2 ** (b - 1) < L ** g <= 2 ** b          # b is the fewest bits holding L**g values
        assert b / g == pytest.approx(O.pages_code_bits(L))


def test_row_bits_counted_by_hand():
    # 6 levels: 25 groups of 13 bits + 3 digits (216 values) in 8 bits
    assert O.pages_row_bits(6) == 25 * 13 + 8 == 333
    # 5 levels: 42 groups of 7 bits + 2 digits (25 values) in 5 bits
    assert O.pages_row_bits(5) == 42 * 7 + 5 == 299
    assert O.pages_row_bits(8) == 384 and O.pages_row_bits(4) == 256
    for L in range(2, 17):
        groups = O.pages_groups(L)
        assert sum(k for _, k, _, _ in groups) == 128
        assert groups[-1][3] + groups[-1][2] == O.pages_row_bits(L)


def _brute_unpack(stream_bytes, n, L, D=128):
    """Independent reader: walk the bit stream one bit at a time with Python ints."""
    bits = []
    for byte in stream_bytes:
        for i in range(8):
            bits.append((int(byte) >> i) & 1)
    g, b = O.pages_group(L)
    out = []
    pos = 0
    for _ in range(n):
        row = []
        left = D
        while left > 0:
            k = min(g, left)
            nb = (L ** k - 1).bit_length()
            val = sum(bits[pos + i] << i for i in range(nb))
            pos += nb
            for _ in range(k):
                row.append(val % L)
                val //= L
            left -= k
        out.append(row)
    return np.array(out, dtype=np.uint8)


@pytest.mark.parametrize("L", [3, 4, 5, 6, 7, 8, 11, 16])
def test_pack_matches_brute_force_reader_and_round_trips(L):
    rng = np.random.default_rng(700 + L)
    codes = rng.integers(0, L, (9, 128)).astype(np.uint8)
    codes[0] = L - 1
    codes[1] = 0
    stream = O.pack_rows_pages(codes, L)
    assert stream.dtype == np.uint8 and stream.size == (9 * O.pages_row_bits(L) + 7) // 8
    assert np.array_equal(_brute_unpack(stream, 9, L), codes)
    assert np.array_equal(O.unpack_rows_pages(stream, 9, L), codes)


def test_first_group_bits_by_hand():
    # digits 1, 2, 3, 4, 5 of one 6-level row: value 1 + 2*6 + 3*36 + 4*216 + 5*1296 = 7465
    codes = np.zeros((2, 128), np.uint8)
    codes[0, :5] = [1, 2, 3, 4, 5]
    codes[1, 0] = 1                              # row 1 starts at stream bit 333
    s = O.pack_rows_pages(codes, 6)
    v = int.from_bytes(s.tobytes(), "little")
    assert v & 0x1FFF == 7465
    assert (v >> 333) & 0x1FFF == 1
    assert v & ~((0x1FFF) | (0x1FFF << 333)) == 0


def _golden_rows():
    rows = []
    for line in open(os.path.join(GOLDEN, "storage_table.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([x.strip() for x in line.split("|")])
    return rows


def test_printed_compressions_from_stored_bytes():
    # affine rows of the printed table (two 16-bit scalars per row): the byte
    # count of a real pool in this layout gives the printed compression
    n = 4096
    checked = 0
    for name, mix, meta, eff, comp, _ in _golden_rows():
        if meta != "2" or comp == "-":
            continue
        parts = [(int(a), float(b)) for a, b in (p.split(":") for p in mix.split(","))]
        total = sum(O.pages_layout_bytes(int(round(n * f)), L) for L, f in parts)
        assert round(16 * 128 * n / 8 / total, 1) == float(comp), name
        checked += 1
    assert checked == 5


def test_fp16_scalars_and_dequantization_bound():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((300, 128)) * rng.lognormal(0, 1, (300, 1))).astype(np.float16)
    for L in (5, 6):
        c, mn, sc, _ = O.quantize_rows(x, L)
        mn16, sc16 = O.pages_meta(mn, sc)
        assert np.array_equal(mn16.astype(np.float32), mn)        # the min of fp16 values is an fp16 value
        assert np.all(np.abs(sc16.astype(np.float64) - sc) <= np.abs(sc) * 2.0 ** -11)
        xhat = mn16.astype(np.float64)[:, None] + c * sc16.astype(np.float64)[:, None]
        err = np.abs(x.astype(np.float64) - xhat)
        bound = sc[:, None] * (0.5 + 2 ** -20 + (L - 1) * 2.0 ** -11) + 2 ** -22 * np.abs(mn)[:, None]
        assert np.all(err <= bound)
