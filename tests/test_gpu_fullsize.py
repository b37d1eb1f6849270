"""Parity at the full workload sizes, in the launch configuration bench.py uses.

The oracle cannot redo a whole 32-layer cache in seconds, so each test checks
every output that is cheap to check exactly (all masks, all counts, key-L2
scores of whole layers) and samples the rest: whole (sequence, layer, head)
slabs of the pools (bit-exact, every row) and decode outputs of sampled KV
heads (float64 oracle on its own pools built from the same inputs).

Every oracle input is a synthetic input or an oracle output: the masks the
oracle quantizes with come from the oracle's own scores.  Where the GPU mask
comes from attention-mass scores (checked within tolerance), it may differ from
the oracle's only at tokens within that tolerance of the threshold; the pools
are then checked on a GPU quantize run with the oracle's mask.
"""
import numpy as np
import pytest
import torch

from inputs import synth
from oracle import semkv_oracle as O
from tests.gpu_common import (SCORE_ATOL, SCORE_RTOL, check_attention, check_mask_near_threshold, kv_mod,
                              to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cache_for(kv, wl, r_ppm, T_cap, L_high=None, L_low=None, gen=0, block=128):
    L_high = wl.L_high if L_high is None else L_high
    L_low = wl.L_low if L_low is None else L_low
    nh = kv.semkv_num_high(T_cap, r_ppm)
    extra = kv.semkv_num_high(block, r_ppm) * (gen // block + 2)
    return kv.MixedCache(wl.B, wl.Lyr, wl.H, wl.H_q, L_high, L_low, r_ppm, nh + extra + 16,
                         T_cap - nh + block * (gen // block + 2) + 16, block=block)


def _check_slab(cache, x_slab, mask, b, l, h, which, L_high, L_low):
    """Every pool row of one (sequence, layer, head) of K or V, bit-exact."""
    ph, pl, _ = O.quantize_slab(x_slab, mask, L_high, L_low)
    nh, nl = int(cache.n_high[b]), int(cache.n_low[b])
    for pool, n, words, meta in ((ph, nh, getattr(cache, which + "_high"), getattr(cache, which + "_high_meta")),
                                 (pl, nl, getattr(cache, which + "_low"), getattr(cache, which + "_low_meta"))):
        assert pool.words.shape[0] == n
        if n == 0:
            continue
        assert np.array_equal(to_np(words[b, l, h, :n]).view(np.uint32), pool.words), (which, b, l, h)
        gm = to_np(meta[b, l, h, :n])
        assert np.array_equal(gm[:, 0].view(np.uint32), pool.mn.view(np.uint32)), (which, b, l, h)
        assert np.array_equal(gm[:, 1].view(np.uint32), pool.scale.view(np.uint32)), (which, b, l, h)


def _oracle_decode_head(ks, vs, mask, q_heads, L_high, L_low, buf_k=None, buf_v=None):
    """float64 decode of the query heads of one KV head from the oracle's own pools."""
    kk, vv = [], []
    for x, acc in ((ks, kk), (vs, vv)):
        ph, pl, _ = O.quantize_slab(x, mask, L_high, L_low)
        for p, L in ((ph, L_high), (pl, L_low)):
            if p.words.shape[0]:
                acc.append(O.dequantize(O.unpack_rows(p.words, L), p.mn, p.scale))
    if buf_k is not None and buf_k.shape[0]:
        kk.append(buf_k.astype(np.float64))
        vv.append(buf_v.astype(np.float64))
    return O.decode_attn(q_heads, [np.concatenate(kk)], [np.concatenate(vv)])


# ------------------------------------------------------------------ llama prefill
def test_llama8b_prefill_full_size():
    kv = kv_mod()
    wl = synth.LLAMA_PREFILL
    B, Lyr, H, H_q, T, w = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T, wl.w
    k, v = synth.kv(wl, 0, DEV)
    q_win = synth.q_window(wl, 0, DEV)
    seq_len = synth.seq_lens(wl, 0).to(DEV)
    score = torch.empty((B, T), device=DEV)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, Lyr - 1], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
    mask = torch.empty((B, T), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    torch.cuda.synchronize()
    nh = O.num_high(T, wl.r_ppm)
    s_ref = O.score_attn_mass(to_np(k[0, Lyr - 1]), to_np(q_win[0]), T)
    assert np.all(np.abs(to_np(score)[0] - s_ref) <= SCORE_RTOL * np.abs(s_ref) + SCORE_ATOL)
    m = O.select_mask(s_ref.astype(np.float32), nh)
    flips = check_mask_near_threshold(to_np(mask)[0], s_ref, m, nh)
    print(f"[mask flips] {wl.name} seq 0: {flips} of {T} tokens differ from the oracle's mask, "
          f"all within the score tolerance of the threshold")

    # quantize + decode of the whole cache, on the oracle's mask
    mask.copy_(torch.from_numpy(m)[None])
    cache = _cache_for(kv, wl, wl.r_ppm, T)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    q = synth.decode_query(wl, 0, DEV)
    out = torch.empty_like(q)
    kv.semkv_decode_attn(cache, 0, Lyr, q, out)
    torch.cuda.synchronize()
    assert cache.status_flags() == 0
    assert int(cache.n_high[0]) == nh and int(cache.n_low[0]) == T - nh
    qn = to_np(q)
    G = H_q // H
    for l, h in ((0, 0), (13, 5), (Lyr - 1, 7)):
        ks, vs = to_np(k[0, l, h]), to_np(v[0, l, h])
        _check_slab(cache, ks, m, 0, l, h, "k", wl.L_high, wl.L_low)
        _check_slab(cache, vs, m, 0, l, h, "v", wl.L_high, wl.L_low)
        ref = _oracle_decode_head(ks, vs, m, qn[0, l, h * G:(h + 1) * G], wl.L_high, wl.L_low)
        check_attention(to_np(out[0, l, h * G:(h + 1) * G]), ref)


# ------------------------------------------------------------------ mistral long context, r sweep
def test_mistral7b_long_context_r_sweep():
    kv = kv_mod()
    wl = synth.MISTRAL_LONG
    B, Lyr, H, H_q, T = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T
    k, v = synth.kv(wl, 0, DEV)
    seq_len = synth.seq_lens(wl, 0).to(DEV)
    score = torch.empty((B, T), device=DEV)
    kv.semkv_score(kv.SCORE_KEY_L2, k[:, Lyr - 1], k.stride(0), None, seq_len, B, T, H, H_q, 64, score)
    torch.cuda.synchronize()
    s = to_np(score)[0]
    s_ref = O.score_key_l2(to_np(k[0, Lyr - 1]))
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32))
    q = synth.decode_query(wl, 0, DEV)
    qn = to_np(q)
    mask = torch.empty((B, T), dtype=torch.uint8, device=DEV)
    for r_ppm in synth.R_SWEEP_PPM:
        kv.semkv_select(score, seq_len, r_ppm, mask)
        m = O.select_mask(s_ref, O.num_high(T, r_ppm))
        assert np.array_equal(to_np(mask)[0], m), r_ppm
        if r_ppm not in (100_000, 900_000):
            continue
        cache = _cache_for(kv, wl, r_ppm, T)
        kv.semkv_quantize(cache, k, v, seq_len, mask)
        out = torch.empty_like(q)
        kv.semkv_decode_attn(cache, 0, Lyr, q, out)
        torch.cuda.synchronize()
        assert cache.status_flags() == 0
        assert int(cache.n_high[0]) == O.num_high(T, r_ppm)
        for l, h in ((3, 2), (Lyr - 1, 6)):
            ks, vs = to_np(k[0, l, h]), to_np(v[0, l, h])
            _check_slab(cache, ks, m, 0, l, h, "k", wl.L_high, wl.L_low)
            _check_slab(cache, vs, m, 0, l, h, "v", wl.L_high, wl.L_low)
            G = H_q // H
            ref = _oracle_decode_head(ks, vs, m, qn[0, l, h * G:(h + 1) * G], wl.L_high, wl.L_low)
            check_attention(to_np(out[0, l, h * G:(h + 1) * G]), ref)
        del cache


# ------------------------------------------------------------------ level sweep
@pytest.mark.parametrize("L_high,L_low", synth.LEVEL_PAIRS)
def test_level_sweep_full_size(L_high, L_low):
    kv = kv_mod()
    wl = synth.LEVEL_SWEEP
    B, Lyr, H, H_q, T, w = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T, wl.w
    k, v = synth.kv(wl, L_high * 17 + L_low, DEV)
    q_win = synth.q_window(wl, 0, DEV)
    seq_len = synth.seq_lens(wl, 0).to(DEV)
    score = torch.empty((B, T), device=DEV)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, 0], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
    mask = torch.empty((B, T), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    torch.cuda.synchronize()
    nh = O.num_high(T, wl.r_ppm)
    assert to_np(mask).sum(axis=1).tolist() == [nh] * B
    # sampled sequences: oracle score and mask, GPU mask near-threshold agreement
    samples = (0, B - 1)
    m_all = to_np(mask).copy()
    for b in samples:
        s_ref = O.score_attn_mass(to_np(k[b, 0]), to_np(q_win[b]), T)
        assert np.all(np.abs(to_np(score)[b] - s_ref) <= SCORE_RTOL * np.abs(s_ref) + SCORE_ATOL)
        m_all[b] = O.select_mask(s_ref.astype(np.float32), nh)
        flips = check_mask_near_threshold(to_np(mask)[b], s_ref, m_all[b], nh)
        print(f"[mask flips] {wl.name} {L_high}/{L_low} seq {b}: {flips} of {T} tokens differ from the "
              f"oracle's mask, all within the score tolerance of the threshold")
    mask.copy_(torch.from_numpy(m_all))
    cache = _cache_for(kv, wl, wl.r_ppm, T, L_high, L_low)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    q = synth.decode_query(wl, 1, DEV)
    out = torch.empty_like(q)
    kv.semkv_decode_attn(cache, 0, 1, q, out)
    torch.cuda.synchronize()
    assert cache.status_flags() == 0
    assert to_np(cache.n_high).tolist() == [nh] * B
    qn = to_np(q)
    G = H_q // H
    for b, h in ((samples[0], 0), (samples[1], H - 1)):
        ks, vs = to_np(k[b, 0, h]), to_np(v[b, 0, h])
        _check_slab(cache, ks, m_all[b], b, 0, h, "k", L_high, L_low)
        _check_slab(cache, vs, m_all[b], b, 0, h, "v", L_high, L_low)
        ref = _oracle_decode_head(ks, vs, m_all[b], qn[b, 0, h * G:(h + 1) * G], L_high, L_low)
        check_attention(to_np(out[b, 0, h * G:(h + 1) * G]), ref)


# ------------------------------------------------------------------ generation, block-exact
def test_generation_full_size():
    """B=16 prompts ~U[4096,16384], 512 generated tokens appended one per step with
    a key-L2 score of the new token at the last layer, decode over all 32 layers
    every step.  Sampled slabs are replayed by the oracle: the prompt quantized
    with the oracle's own attention-mass mask (fed to the GPU for those
    sequences), then every full block ranked by the oracle's own key-L2 scores."""
    kv = kv_mod()
    wl = synth.GENERATION
    B, Lyr, H, H_q, T, w = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T, wl.w
    lens = synth.seq_lens(wl, 0)
    seq_len = lens.to(DEV)
    k, v = synth.kv(wl, 0, DEV)
    q_win = synth.q_window(wl, 0, DEV)
    score = torch.empty((B, T), device=DEV)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, Lyr - 1], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
    mask = torch.empty((B, T), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    torch.cuda.synchronize()
    samples = ((0, 0, 0), (9, Lyr - 1, 5))                    # (sequence, layer, KV head)
    seqs = sorted({b for b, _, _ in samples})
    m_all = to_np(mask).copy()
    for b in seqs:
        T0 = int(lens[b])
        s_ref = O.score_attn_mass(to_np(k[b, Lyr - 1]), to_np(q_win[b]), T0)
        nh = O.num_high(T0, wl.r_ppm)
        m_all[b, :T0] = O.select_mask(s_ref.astype(np.float32), nh)
        flips = check_mask_near_threshold(to_np(mask)[b, :T0], s_ref, m_all[b, :T0], nh)
        print(f"[mask flips] {wl.name} seq {b}: {flips} of {T0} tokens differ from the oracle's mask, "
              f"all within the score tolerance of the threshold")
    mask.copy_(torch.from_numpy(m_all))
    cache = _cache_for(kv, wl, wl.r_ppm, T, gen=wl.gen_steps)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    prompt = {(b, l, h): (to_np(k[b, l, h, :int(lens[b])]), to_np(v[b, l, h, :int(lens[b])])) for b, l, h in samples}
    del k, v
    torch.cuda.empty_cache()

    new_k = {key: [] for key in samples}
    new_v = {key: [] for key in samples}
    new_klast = {b: [] for b in seqs}                          # new key at the last layer, all heads
    out = torch.empty((B, Lyr, H_q, 128), dtype=torch.float16, device=DEV)
    s_new = torch.empty((B, 1), device=DEV)
    ones = torch.ones(B, dtype=torch.int32, device=DEV)
    check_steps = {5, 127, 128, 300, wl.gen_steps - 1}
    G = H_q // H
    for step in range(wl.gen_steps):
        kn, vn, qn = synth.new_tokens(wl, 0, step, DEV)
        # indicator of the new token: key-L2 at the last layer (O(1) per step)
        kv.semkv_score(kv.SCORE_KEY_L2, kn[:, Lyr - 1], kn.stride(0), None, ones, B, 1, H, H_q, w, s_new)
        kv.semkv_append_block(cache, kn, vn, s_new, 1)
        kv.semkv_decode_attn(cache, 0, Lyr, qn, out)
        for b, l, h in samples:
            new_k[(b, l, h)].append(to_np(kn[b, l, h, 0]))
            new_v[(b, l, h)].append(to_np(vn[b, l, h, 0]))
        for b in seqs:
            klast = to_np(kn[b, Lyr - 1, :, 0])                 # [H][128]
            new_klast[b].append(klast)
            s_ref = O.score_key_l2(klast[:, None, :])[0]
            assert to_np(s_new)[b, 0] == s_ref                  # bit-exact indicator
        if step in check_steps:
            torch.cuda.synchronize()
            assert cache.status_flags() == 0
            o = to_np(out)
            q_np = to_np(qn)
            for b, l, h in samples:
                (ks, vs, mk), (bk, bv) = _replay(prompt[(b, l, h)], m_all[b, :int(lens[b])], new_k[(b, l, h)],
                                                 new_v[(b, l, h)], new_klast[b], wl)
                ref = _oracle_decode_head(ks, vs, mk, q_np[b, l, h * G:(h + 1) * G], wl.L_high, wl.L_low, bk, bv)
                check_attention(o[b, l, h * G:(h + 1) * G], ref)
    torch.cuda.synchronize()
    n_blocks = wl.gen_steps // 128
    for b in range(B):
        assert int(cache.n_high[b]) == O.num_high(int(lens[b]), wl.r_ppm) + n_blocks * O.num_high(128, wl.r_ppm)
        assert int(cache.n_low[b]) + int(cache.n_high[b]) == int(lens[b]) + wl.gen_steps
    # every pool row of the sampled slabs: the pools hold the prompt's rows, then each block's
    for b, l, h in samples:
        (ks, vs, mk), (bk, _) = _replay(prompt[(b, l, h)], m_all[b, :int(lens[b])], new_k[(b, l, h)],
                                        new_v[(b, l, h)], new_klast[b], wl)
        assert bk.shape[0] == 0
        _check_slab(cache, ks, mk, b, l, h, "k", wl.L_high, wl.L_low)
        _check_slab(cache, vs, mk, b, l, h, "v", wl.L_high, wl.L_low)


def _replay(prompt_kv, pmask, nk, nv, nklast, wl):
    """Oracle state of one slab after len(nk) appended tokens:
    ((K rows, V rows, mask) of the quantized part, (K, V) of the FP16 block).
    Each full block is ranked by the oracle's key-L2 of the new keys."""
    pk, pv = prompt_kv
    n = len(nk)
    full = (n // 128) * 128
    masks = [pmask]
    for blk in range(n // 128):
        kl = np.stack(nklast[blk * 128:(blk + 1) * 128], axis=1)       # [H][128 tokens][128]
        masks.append(O.select_mask(O.score_key_l2(kl), O.num_high(128, wl.r_ppm)))
    nk_a = np.stack(nk) if n else np.zeros((0, 128), np.float16)
    nv_a = np.stack(nv) if n else np.zeros((0, 128), np.float16)
    return ((np.concatenate([pk, nk_a[:full]]), np.concatenate([pv, nv_a[:full]]), np.concatenate(masks)),
            (nk_a[full:], nv_a[full:]))
