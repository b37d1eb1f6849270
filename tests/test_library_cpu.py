"""Host-side checks of libsemkv.so that need no GPU: it loads, exports every
symbol include/semkv.h declares, its host helpers agree with the oracle, and
bad arguments are rejected before anything is launched."""
import ctypes
import os
import re

import pytest

from oracle import semkv_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kv():
    import __graft_entry__
    __graft_entry__.build()
    import kv_cache_mixed_b200 as kv
    return kv


def test_library_exports_every_declared_symbol(kv):
    hdr = open(os.path.join(ROOT, "include", "semkv.h")).read()
    declared = sorted(set(re.findall(r"\b(semkv_[a-z_0-9]+)\s*\(", hdr)))
    assert len(declared) >= 14
    lib = ctypes.CDLL(kv.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(kv.EXPORTED) == declared


def test_host_helpers_match_oracle(kv):
    for L in range(2, 17):
        assert kv.semkv_digits_per_word(L) == O.digits_per_word(L)
        assert kv.semkv_words_per_row(L) == O.words_per_row(L)
    assert kv.semkv_digits_per_word(1) == -1 and kv.semkv_digits_per_word(17) == -1
    for n, r in [(0, 0), (32768, 100_000), (131072, 250_000), (128, 500_000), (77, 999_999), (5, 1_000_000)]:
        assert kv.semkv_num_high(n, r) == O.num_high(n, r)
    assert kv.semkv_num_high(-1, 5) == -1 and kv.semkv_num_high(5, 1_000_001) == -1
    assert "sm_100a" in kv.semkv_version()
    # storage sizes of both layouts (the pages' layout: rows back to back at bit granularity)
    for L in range(2, 17):
        assert kv.semkv_row_bits(kv.LAYOUT_WORDS, L) == 32 * O.words_per_row(L)
        assert kv.semkv_pool_words(kv.LAYOUT_WORDS, L, 48) == 48 * O.words_per_row(L)
        if L in (9, 12, 14, 15):
            assert kv.semkv_row_bits(kv.LAYOUT_PAGES, L) == -1
            continue
        assert kv.semkv_row_bits(kv.LAYOUT_PAGES, L) == O.pages_row_bits(L)
        assert kv.semkv_pool_words(kv.LAYOUT_PAGES, L, 48) * 4 >= (48 * O.pages_row_bits(L) + 7) // 8
        assert kv.semkv_pool_words(kv.LAYOUT_PAGES, L, 48) % 4 == 0
    assert kv.semkv_row_bits(2, 6) == -1 and kv.semkv_pool_words(kv.LAYOUT_PAGES, 6, -1) == -1


def test_invalid_arguments_rejected_before_launch(kv):
    b = kv.binding
    INVALID, UNSUP, WS = 1, 2, 3
    # null cache
    assert b._lib_quant(None, None, None, 16, None, None, None, 0, None, None) == INVALID
    assert b._lib_decode(None, 0, 1, None, None, 1.0, None, 0, None, None) == INVALID
    assert b._lib_append(None, None, None, None, 1, 0, None, 0, None, None) == INVALID
    # a cache with D != 128, bad levels, unaligned pointers, bad capacities
    def cache(**kw):
        base = dict(B=1, n_layers=1, H=1, H_q=4, D=128, L_high=6, L_low=5, r_ppm=500_000, cap_high=16,
                    cap_low=16, block=128, buf_len=0, rotate=0, layout=0)
        base.update(kw)
        names = ("B", "n_layers", "H", "H_q", "D", "L_high", "L_low", "r_ppm", "cap_high", "cap_low", "block",
                 "buf_len", "rotate", "layout")
        c = b.SemkvCache(*[base[k] for k in names])
        for f, _ in b.SemkvCache._fields_[len(names):]:
            setattr(c, f, 0x10000)
        return c
    for kw, want in [(dict(D=64), UNSUP), (dict(L_high=17), UNSUP), (dict(L_low=1), UNSUP),
                     (dict(H_q=3, H=2), INVALID), (dict(H_q=36, H=4), UNSUP), (dict(r_ppm=-1), INVALID),
                     (dict(cap_high=17), INVALID), (dict(block=0), INVALID), (dict(buf_len=128), INVALID),
                     (dict(rotate=2), INVALID), (dict(rotate=1, H_q=8, H=1), UNSUP),
                     (dict(layout=2), INVALID), (dict(layout=1, L_high=12), UNSUP),
                     (dict(layout=1, L_low=9), UNSUP), (dict(layout=1, rotate=1), UNSUP)]:
        c = cache(**kw)
        assert b._lib_decode(ctypes.byref(c), 0, 1, ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 1.0,
                             ctypes.c_void_p(0x10000), 1 << 20, None, None) == want, kw
    c = cache()
    c.k_low = 0x10008                              # misaligned pool
    assert b._lib_quant(ctypes.byref(c), ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 16,
                        ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 1 << 20,
                        None, None) == INVALID
    c = cache()
    # workspace too small
    assert b._lib_quant(ctypes.byref(c), ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 16,
                        ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 8,
                        None, None) == WS
    # decode: layer range, bad scale
    assert b._lib_decode(ctypes.byref(c), 1, 1, ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 1.0,
                         ctypes.c_void_p(0x10000), 1 << 20, None, None) == INVALID
    assert b._lib_decode(ctypes.byref(c), 0, 1, ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), -1.0,
                         ctypes.c_void_p(0x10000), 1 << 20, None, None) == INVALID
    # decode with score accumulation: the scoring layer must be one of the decoded layers
    assert b._lib_decode_acc(ctypes.byref(c), 0, 1, 1, ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 1.0,
                             ctypes.c_void_p(0x10000), 1 << 20, None, None) == INVALID
    assert b._lib_decode_acc(ctypes.byref(c), 0, 1, -1, ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10000), 1.0,
                             ctypes.c_void_p(0x10000), 1 << 20, None, None) == INVALID
    # append: negative n, unknown flag
    assert b._lib_append(ctypes.byref(c), None, None, None, -1, 0, ctypes.c_void_p(0x10000), 1 << 20,
                         None, None) == INVALID
    assert b._lib_append(ctypes.byref(c), None, None, None, 0, 2, ctypes.c_void_p(0x10000), 1 << 20,
                         None, None) == INVALID
    # score / select argument checks
    assert b._lib_score(7, ctypes.c_void_p(0x10000), 1 << 20, None, ctypes.c_void_p(0x10000), 1, 16, 1, 4,
                        128, 4, ctypes.c_void_p(0x10000), None, 0, None, None) == INVALID
    assert b._lib_score(1, ctypes.c_void_p(0x10000), 1 << 20, None, ctypes.c_void_p(0x10000), 1, 16, 1, 4,
                        64, 4, ctypes.c_void_p(0x10000), None, 0, None, None) == UNSUP
    assert b._lib_score(0, ctypes.c_void_p(0x10000), 1 << 20, ctypes.c_void_p(0x10000),
                        ctypes.c_void_p(0x10000), 1, 16, 1, 4, 128, 4, ctypes.c_void_p(0x10000), None, 0,
                        None, None) == WS
    assert b._lib_select(ctypes.c_void_p(0x10000), 16, None, 17, 1, 16, 500_000, ctypes.c_void_p(0x10000), 16,
                         None, 0, None, None) == INVALID
    assert b._lib_select(ctypes.c_void_p(0x10000), 16, None, 4, 1, 16, 2_000_000, ctypes.c_void_p(0x10000), 16,
                         None, 0, None, None) == INVALID
