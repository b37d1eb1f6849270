"""Device status flags, the bounded-wait timeout path and output canaries,
through the C ABI (GPU).

* SEMKV_FLAG_SEQLEN: a sequence whose length exceeds T_max is skipped by every
  call that takes lengths (score, select, quantize); the other sequences stay
  bit-exact against the oracle, and nothing is written outside the slots in
  use (pools are filled with a sentinel first and checked after).
* SEMKV_FLAG_TIMEOUT: the testing aid semkv_set_first_copy_wait_polls(0) makes
  the first wait of every warp's copy ring give up at once.  The call must
  return with the flag set after draining its copies, and the very next call
  with the default bound must be exact again (the GPU stays usable).
"""
import numpy as np
import pytest
import torch

from inputs import synth
from oracle import semkv_oracle as O
from tests.gpu_common import check_attention, kv_mod, new_cache, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENTINEL = 0x5A5A5A5A


def _fill_sentinel(cache):
    for t in (cache.k_high, cache.v_high, cache.k_low, cache.v_low):
        t.fill_(SENTINEL)
    for t in (cache.k_high_meta, cache.v_high_meta, cache.k_low_meta, cache.v_low_meta):
        t.view(torch.int32).fill_(SENTINEL)


def _pools(cache):
    return ((cache.k_high, cache.k_high_meta, cache.n_high, "k"), (cache.v_high, cache.v_high_meta, cache.n_high, "v"),
            (cache.k_low, cache.k_low_meta, cache.n_low, "k"), (cache.v_low, cache.v_low_meta, cache.n_low, "v"))


def _check_canaries(cache):
    """Every slot at or past n of its class, for every (sequence, layer, head), still holds the sentinel."""
    for words, meta, cnt, _ in _pools(cache):
        n = to_np(cnt)
        w = to_np(words).view(np.uint32)
        m = to_np(meta.view(torch.int32)).view(np.uint32)
        for b in range(w.shape[0]):
            assert np.all(w[b, :, :, n[b]:] == SENTINEL), b
            assert np.all(m[b, :, :, n[b]:] == SENTINEL), b


def _compare_seq(cache, k, v, mask, b, T, L_high, L_low):
    m = mask[:T]
    nh = int(to_np(cache.n_high)[b])
    nl = int(to_np(cache.n_low)[b])
    assert nh == int(m.sum()) and nl == T - nh
    kk, vv = to_np(k[b]), to_np(v[b])
    for l in range(k.shape[1]):
        for h in range(k.shape[2]):
            for x, (wh, wl_, mh, ml) in ((kk, (cache.k_high, cache.k_low, cache.k_high_meta, cache.k_low_meta)),
                                         (vv, (cache.v_high, cache.v_low, cache.v_high_meta, cache.v_low_meta))):
                ph, pl, _ = O.quantize_slab(x[l, h, :T], m, L_high, L_low)
                for pool, words, meta, n in ((ph, wh, mh, nh), (pl, wl_, ml, nl)):
                    assert np.array_equal(to_np(words[b, l, h, :n]).view(np.uint32), pool.words)
                    gm = to_np(meta[b, l, h, :n])
                    assert np.array_equal(gm[:, 0].view(np.uint32), pool.mn.view(np.uint32))
                    assert np.array_equal(gm[:, 1].view(np.uint32), pool.scale.view(np.uint32))


def test_seqlen_flag_skips_only_that_sequence():
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=3, Lyr=2, H=2, H_q=8, T=300)
    k, v = synth.kv(wl, 1, DEV)
    q_win = synth.q_window(wl, 1, DEV)
    lens = [257, 301, 90]                         # sequence 1 is one past T_max
    seq_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)

    # key-L2 score: flagged, sequence 1 all zero, the others bit-exact
    score = torch.full((3, 300), 7.0, device=DEV)
    kv.semkv_score(kv.SCORE_KEY_L2, k[:, 1], k.stride(0), None, seq_len, 3, 300, 2, 8, 64, score, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == kv.FLAG_SEQLEN
    s = to_np(score)
    assert np.all(s[1] == 0)
    for b in (0, 2):
        assert np.array_equal(s[b, :lens[b]], O.score_key_l2(to_np(k[b, 1, :, :lens[b]])))
        assert np.all(s[b, lens[b]:] == 0)

    # attention-mass score: flagged, sequence 1 all zero
    status.zero_()
    am = torch.full((3, 300), 7.0, device=DEV)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, 1], k.stride(0), q_win, seq_len, 3, 300, 2, 8, 64, am, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & kv.FLAG_SEQLEN
    assert np.all(to_np(am)[1] == 0)

    # select: flagged, mask of sequence 1 all zero, the others exact
    status.zero_()
    mask = torch.full((3, 300), 9, dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == kv.FLAG_SEQLEN
    mk = to_np(mask)
    assert np.all(mk[1] == 0)
    for b in (0, 2):
        assert np.array_equal(mk[b, :lens[b]], O.select_mask(s[b, :lens[b]], O.num_high(lens[b], wl.r_ppm)))
        assert np.all(mk[b, lens[b]:] == 0)

    # quantize: flagged; sequence 1 writes nothing and keeps counts 0; 0 and 2 bit-exact
    cache = new_cache(3, 2, 2, 8, 6, 5, wl.r_ppm, 300)
    _fill_sentinel(cache)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    torch.cuda.synchronize()
    assert cache.status_flags() == kv.FLAG_SEQLEN
    assert to_np(cache.n_high)[1] == 0 and to_np(cache.n_low)[1] == 0
    for b in (0, 2):
        _compare_seq(cache, k, v, mk[b], b, lens[b], 6, 5)
    _check_canaries(cache)


def test_quantize_timeout_path_flags_and_recovers():
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=2, Lyr=2, H=2, H_q=8, T=520)
    k, v = synth.kv(wl, 2, DEV)
    score = synth.uniform_score(wl, 2, DEV)
    seq_len = torch.tensor([520, 333], dtype=torch.int32, device=DEV)
    mask = torch.zeros((2, 520), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    cache = new_cache(2, 2, 2, 8, 6, 5, wl.r_ppm, 520)
    kv.semkv_set_first_copy_wait_polls(0)
    try:
        kv.semkv_quantize(cache, k, v, seq_len, mask)
    finally:
        kv.semkv_set_first_copy_wait_polls(-1)
    torch.cuda.synchronize()
    assert cache.status_flags() & kv.FLAG_TIMEOUT
    # the next call, with the default bound, is exact
    fresh = new_cache(2, 2, 2, 8, 6, 5, wl.r_ppm, 520)
    _fill_sentinel(fresh)
    kv.semkv_quantize(fresh, k, v, seq_len, mask)
    torch.cuda.synchronize()
    assert fresh.status_flags() == 0
    mk = to_np(mask)
    for b, T in ((0, 520), (1, 333)):
        _compare_seq(fresh, k, v, mk[b], b, T, 6, 5)
    _check_canaries(fresh)


def test_decode_timeout_path_flags_and_recovers():
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=2, Lyr=2, H=2, H_q=8, T=700)
    k, v = synth.kv(wl, 3, DEV)
    score = synth.uniform_score(wl, 3, DEV)
    seq_len = torch.tensor([700, 411], dtype=torch.int32, device=DEV)
    mask = torch.zeros((2, 700), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    cache = new_cache(2, 2, 2, 8, 6, 5, wl.r_ppm, 700)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    q = synth.decode_query(wl, 3, DEV)
    out = torch.zeros_like(q)
    torch.cuda.synchronize()
    assert cache.status_flags() == 0
    kv.semkv_set_first_copy_wait_polls(0)
    try:
        kv.semkv_decode_attn(cache, 0, 2, q, out)
    finally:
        kv.semkv_set_first_copy_wait_polls(-1)
    torch.cuda.synchronize()
    assert cache.status_flags() & kv.FLAG_TIMEOUT
    cache.status.zero_()
    kv.semkv_decode_attn(cache, 0, 2, q, out)
    torch.cuda.synchronize()
    assert cache.status_flags() == 0
    mk = to_np(mask)
    kk, vv, qq = to_np(k), to_np(v), to_np(q)
    ref = np.zeros(q.shape)
    for b, T in ((0, 700), (1, 411)):
        for l in range(2):
            keys, vals = [], []
            for h in range(2):
                kh, vh = [], []
                for x, acc in ((kk, kh), (vv, vh)):
                    ph, pl, _ = O.quantize_slab(x[b, l, h, :T], mk[b, :T], 6, 5)
                    for p, L in ((ph, 6), (pl, 5)):
                        acc.append(O.dequantize(O.unpack_rows(p.words, L), p.mn, p.scale))
                keys.append(np.concatenate(kh))
                vals.append(np.concatenate(vh))
            ref[b, l] = O.decode_attn(qq[b, l], keys, vals)
    check_attention(to_np(out).astype(np.float64), ref)


def test_decode_writes_only_its_outputs():
    """Canaries around the decode outputs: a sentinel tail after `out` stays, the
    pools and the query are read-only, and with score accumulation only the
    FP16 block's first buf_len entries of buf_score change."""
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=2, Lyr=3, H=2, H_q=8, T=300)
    k, v = synth.kv(wl, 6, DEV)
    score = synth.uniform_score(wl, 6, DEV)
    seq_len = torch.tensor([300, 177], dtype=torch.int32, device=DEV)
    mask = torch.zeros((2, 300), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    cache = new_cache(2, 3, 2, 8, 6, 5, wl.r_ppm, 300, block=16)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    kn, vn, _ = synth.new_tokens(wl, 6, 0, DEV, n=5)
    kv.semkv_append_block(cache, kn, vn, torch.rand((2, 5), device=DEV), 5)
    cache.buf_score[:, 5:].fill_(-7.0)                       # entries past buf_len
    pools_before = [t.clone() for t in (cache.k_high, cache.v_high, cache.k_low, cache.v_low,
                                        cache.k_high_meta, cache.v_high_meta, cache.k_low_meta, cache.v_low_meta)]
    q = synth.decode_query(wl, 6, DEV, n_layers=2)
    q_before = q.clone()
    n_out = q.numel()
    out_full = torch.full((n_out + 4096,), 0x5A5A, dtype=torch.int16, device=DEV)
    out = out_full[:n_out].view(torch.float16).view(q.shape)
    kv.semkv_decode_attn_acc(cache, 1, 2, 2, q, out)          # layers 1..2, scores at layer 2
    torch.cuda.synchronize()
    assert cache.status_flags() == 0
    assert torch.all(out_full[n_out:] == 0x5A5A)
    assert torch.isfinite(out).all()
    assert torch.equal(q, q_before)
    for a, b in zip(pools_before, (cache.k_high, cache.v_high, cache.k_low, cache.v_low, cache.k_high_meta,
                                   cache.v_high_meta, cache.k_low_meta, cache.v_low_meta)):
        assert torch.equal(a, b)
    bs = to_np(cache.buf_score)
    assert np.all(bs[:, 5:] == -7.0)
