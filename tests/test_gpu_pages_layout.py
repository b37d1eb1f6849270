"""The pages' own storage layout (SEMKV_LAYOUT_PAGES) on the GPU, through the C ABI.

SemKV, Table 3, Table 5, Table 6 and Fig. 11 count storage as groups of at most
five base-L digits in whole bits plus two 16-bit scalars per row.  The cache
option writes exactly that: one bit stream per (sequence, layer, head) slab
with rows back to back, and fp16 (min, scale).  Checked here:

* quantize: every stream bit of every row and every fp16 scalar equals the
  oracle's (pack_rows_pages, pages_meta) for every supported level and the
  swept pairs, with ragged lengths; the pools start filled with a sentinel, so
  the bits around and after the rows must keep it (rows never clobber their
  neighbours, and no zero-filling is needed);
* decode within the attention tolerance of the float64 oracle on the
  dequantized rows (min16 + code * scale16);
* the generation path: blocks appended one after another in the same stream;
* capacity overflow is flagged and leaves the stream past the capacity alone.
"""
import numpy as np
import pytest
import torch

from inputs import synth
from oracle import semkv_oracle as O
from tests.gpu_common import check_attention, kv_mod, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENT = 0x5A5A5A5A
LEVELS = [(L, L) for L in (2, 3, 4, 5, 6, 7, 8, 10, 11, 13, 16)] + [(6, 5), (5, 4), (8, 6), (16, 8)]


def _cache(kv, B, Lyr, H, H_q, Lh, Ll, r_ppm, cap_h, cap_l, block=128):
    c = kv.MixedCache(B, Lyr, H, H_q, Lh, Ll, r_ppm, cap_h, cap_l, block=block, layout=kv.LAYOUT_PAGES)
    for t in (c.k_high, c.v_high, c.k_low, c.v_low):
        t.fill_(SENT)
    for t in (c.k_high_meta, c.v_high_meta, c.k_low_meta, c.v_low_meta):
        t.view(torch.int16).fill_(0x5A5A)
    return c


def _stream_bits(words_row):
    """uint8 bits (little-endian) of one slab's int32 words."""
    return np.unpackbits(words_row.view(np.uint8), bitorder="little")


def _check_slab(stream_words, meta, x_rows_list, L):
    """The slab's stream holds the rows of x_rows_list (fp16 [n][128] chunks quantized in
    that order, each chunk one quantize call) back to back, then the sentinel."""
    codes, mns, scs = [], [], []
    for xr in x_rows_list:
        c, mn, sc, _ = O.quantize_rows(xr, L)
        codes.append(c)
        mns.append(mn)
        scs.append(sc)
    codes = np.concatenate(codes) if codes else np.zeros((0, 128), np.uint8)
    n = codes.shape[0]
    R = O.pages_row_bits(L)
    want = np.unpackbits(O.pack_rows_pages(codes, L), bitorder="little")[:n * R]
    got = _stream_bits(stream_words)
    assert np.array_equal(got[:n * R], want)
    sent = _stream_bits(np.full(stream_words.shape, SENT, dtype=np.int32))
    assert np.array_equal(got[n * R:], sent[n * R:])          # untouched past the rows
    if n:
        mn16, sc16 = O.pages_meta(np.concatenate(mns), np.concatenate(scs))
        gm = meta[:n].view(np.uint16)
        assert np.array_equal(gm[:, 0], mn16.view(np.uint16))
        assert np.array_equal(gm[:, 1], sc16.view(np.uint16))
    assert np.all(meta[n:].view(np.uint16) == 0x5A5A)
    return codes


def _dequant(codes, meta):
    m = meta[:codes.shape[0]].astype(np.float64)
    return m[:, 0:1] + codes.astype(np.float64) * m[:, 1:2]


@pytest.mark.parametrize("L_high,L_low", LEVELS)
def test_pages_quantize_bit_exact_and_decode(L_high, L_low):
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=2, Lyr=2, H=2, H_q=8, T=333)
    k, v = synth.kv(wl, 900 + L_high * 17 + L_low, DEV)
    score = synth.uniform_score(wl, L_low, DEV)
    lens = [333, 250]
    seq_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
    mask = torch.zeros((2, 333), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    nh = O.num_high(333, wl.r_ppm)
    cache = _cache(kv, 2, 2, 2, 8, L_high, L_low, wl.r_ppm, nh + 16, 333 - nh + 16)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    q = synth.decode_query(wl, 5, DEV)
    out = torch.zeros_like(q)
    kv.semkv_decode_attn(cache, 0, 2, q, out)
    torch.cuda.synchronize()
    assert cache.status_flags() == 0
    mk = to_np(mask)
    kk, vv, qq = to_np(k), to_np(v), to_np(q)
    ref = np.zeros(q.shape)
    for b in range(2):
        T = lens[b]
        m = mk[b, :T]
        hi_idx, lo_idx = np.nonzero(m == 1)[0], np.nonzero(m == 0)[0]
        assert int(to_np(cache.n_high)[b]) == hi_idx.size and int(to_np(cache.n_low)[b]) == lo_idx.size
        for l in range(2):
            keys, vals = [], []
            for h in range(2):
                kh, vh = [], []
                for x, acc, (wh, wl_, mh, ml) in (
                        (kk, kh, (cache.k_high, cache.k_low, cache.k_high_meta, cache.k_low_meta)),
                        (vv, vh, (cache.v_high, cache.v_low, cache.v_high_meta, cache.v_low_meta))):
                    for idx, words, meta, L in ((hi_idx, wh, mh, L_high), (lo_idx, wl_, ml, L_low)):
                        meta_np = to_np(meta[b, l, h])
                        codes = _check_slab(to_np(words[b, l, h]), meta_np, [x[b, l, h, idx]], L)
                        if codes.shape[0]:
                            acc.append(_dequant(codes, meta_np))
                keys.append(np.concatenate(kh))
                vals.append(np.concatenate(vh))
            ref[b, l] = O.decode_attn(qq[b, l], keys, vals)
    check_attention(to_np(out).astype(np.float64), ref)


@pytest.mark.parametrize("L_high,L_low", [(6, 5), (8, 6)])
def test_pages_generation_blocks_share_one_stream(L_high, L_low):
    kv = kv_mod()
    B, Lyr, H, H_q, block = 2, 2, 2, 8, 16
    wl = synth.scaled(synth.TINY, B=B, Lyr=Lyr, H=H, H_q=H_q, T=40)
    cache = _cache(kv, B, Lyr, H, H_q, L_high, L_low, 500_000, 64, 64, block=block)
    chunks, scores = [], []
    for step, n in enumerate((5, 11, 9, 7)):                 # 32 tokens: two full blocks
        kn, vn, _ = synth.new_tokens(wl, 3, step, DEV, n=n)
        sn = torch.rand((B, n), device=DEV, generator=torch.Generator(device=DEV).manual_seed(step))
        kv.semkv_append_block(cache, kn, vn, sn, n)
        chunks.append((to_np(kn), to_np(vn)))
        scores.append(to_np(sn))
    kn, vn, _ = synth.new_tokens(wl, 3, 9, DEV, n=6)
    sn = torch.rand((B, 6), device=DEV, generator=torch.Generator(device=DEV).manual_seed(9))
    kv.semkv_append_block(cache, kn, vn, sn, 6, flags=kv.FLUSH)  # a flushed partial block of 6
    chunks.append((to_np(kn), to_np(vn)))
    scores.append(to_np(sn))
    torch.cuda.synchronize()
    assert cache.status_flags() == 0 and cache.buf_len == 0
    K = np.concatenate([c[0] for c in chunks], axis=3)
    V = np.concatenate([c[1] for c in chunks], axis=3)
    S = np.concatenate(scores, axis=1)
    blocks = [(0, 16), (16, 32), (32, 38)]
    for b in range(B):
        masks = [O.select_mask(S[b, a:e], O.num_high(e - a, 500_000)) for a, e in blocks]
        for l in range(Lyr):
            for h in range(H):
                for x, (wh, wl_, mh, ml) in ((K, (cache.k_high, cache.k_low, cache.k_high_meta, cache.k_low_meta)),
                                             (V, (cache.v_high, cache.v_low, cache.v_high_meta, cache.v_low_meta))):
                    for cls, words, meta, L in ((1, wh, mh, L_high), (0, wl_, ml, L_low)):
                        rows = [x[b, l, h, a:e][m == cls] for (a, e), m in zip(blocks, masks)]
                        _check_slab(to_np(words[b, l, h]), to_np(meta[b, l, h]), rows, L)


def test_pages_capacity_overflow_is_flagged_and_stops_at_capacity():
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=1, Lyr=1, H=1, H_q=4, T=200)
    k, v = synth.kv(wl, 77, DEV)
    seq_len = torch.tensor([200], dtype=torch.int32, device=DEV)
    mask = torch.zeros((1, 200), dtype=torch.uint8, device=DEV)
    mask[0, :100] = 1
    cache = _cache(kv, 1, 1, 1, 4, 6, 5, 500_000, 64, 112)       # 100 high rows into 64 slots
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    torch.cuda.synchronize()
    assert cache.status_flags() & kv.FLAG_CAPACITY
    assert int(cache.n_high[0]) == 64
    kk = to_np(k)
    _check_slab(to_np(cache.k_high[0, 0, 0]), to_np(cache.k_high_meta[0, 0, 0]), [kk[0, 0, 0, :64]], 6)
