"""GPU-vs-oracle parity of every step of the hot path, through the C ABI.

Bit-exact: masks, codes, packed words, fp32 (min, scale), key-L2 scores, counts.
Tolerance: attention-mass scores (1e-4 relative + 1e-6) and decode outputs
(relative L2 <= 1e-3, max-abs <= 5e-3 on fp16 outputs vs the float64 oracle).
Sizes span several tiles and ragged tails; the full workload sizes are in
test_gpu_fullsize.py.
"""
import math

import numpy as np
import pytest
import torch

from inputs import synth
from oracle import semkv_oracle as O
from tests.gpu_common import (MAX_ABS, REL_L2, SCORE_ATOL, SCORE_RTOL, check_attention,
                              check_mask_near_threshold, compare_pools, kv_mod, new_cache, to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _status(cache):
    torch.cuda.synchronize()
    return cache.status_flags()


def _oracle_masks(score, seq_len, r_ppm):
    s = to_np(score)
    return [O.select_mask(s[b, :int(seq_len[b])], O.num_high(int(seq_len[b]), r_ppm)) for b in range(s.shape[0])]


def _prefill(k, v, score, seq_len_t, L_high, L_low, r_ppm, H_q, block=128, gen=0, rotate=False):
    kv = kv_mod()
    B, Lyr, H, T = k.shape[:4]
    mask = torch.zeros((B, T), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len_t, r_ppm, mask)
    cache = new_cache(B, Lyr, H, H_q, L_high, L_low, r_ppm, T, block=block, gen=gen, rotate=rotate)
    kv.semkv_quantize(cache, k, v, seq_len_t, mask)
    return cache, mask


def _oracle_decode_slabs(k, v, masks, seq_len, q, L_high, L_low, buf_k=None, buf_v=None, layer0=0):
    """float64 decode for every (b, layer, query head) from the oracle's own pools."""
    B, nL, H_q, D = q.shape
    H = k.shape[2]
    out = np.zeros((B, nL, H_q, D))
    for b in range(B):
        T = int(seq_len[b])
        for li in range(nL):
            l = layer0 + li
            keys, vals = [], []
            for h in range(H):
                kk, vv = [], []
                for x, acc in ((k, kk), (v, vv)):
                    ph, pl, _ = O.quantize_slab(x[b, l, h, :T], masks[b][:T], L_high, L_low)
                    for p, L in ((ph, L_high), (pl, L_low)):
                        if p.words.shape[0]:
                            acc.append(O.dequantize(O.unpack_rows(p.words, L), p.mn, p.scale))
                if buf_k is not None:
                    kk.append(buf_k[b, l, h].astype(np.float64))
                    vv.append(buf_v[b, l, h].astype(np.float64))
                keys.append(np.concatenate(kk) if kk else np.zeros((0, D)))
                vals.append(np.concatenate(vv) if vv else np.zeros((0, D)))
            out[b, li] = O.decode_attn(q[b, li], keys, vals)
    return out


# ----------------------------------------------------------------- tiny workload
def test_tiny_workload_end_to_end():
    kv = kv_mod()
    wl = synth.TINY
    k, v = synth.kv(wl, 0, DEV)
    score = synth.uniform_score(wl, 0, DEV)
    seq_len = synth.seq_lens(wl, 0).to(DEV)
    cache, mask = _prefill(k, v, score, seq_len, wl.L_high, wl.L_low, wl.r_ppm, wl.H_q)
    masks = _oracle_masks(score, [wl.T], wl.r_ppm)
    assert np.array_equal(to_np(mask)[0], masks[0])
    assert int(masks[0].sum()) == 128
    assert _status(cache) == 0
    kn, vn = to_np(k), to_np(v)
    compare_pools(cache, kn, vn, masks, [wl.T], wl.L_high, wl.L_low)
    q = synth.decode_query(wl, 0, DEV)
    out = torch.empty_like(q)
    kv.semkv_decode_attn(cache, 0, 1, q, out)
    ref = _oracle_decode_slabs(kn, vn, masks, [wl.T], to_np(q), wl.L_high, wl.L_low)
    check_attention(to_np(out), ref)


# ----------------------------------------------------------------- level grid
LEVELS = [(L, L) for L in range(2, 17)] + [(5, 4), (6, 5), (8, 6), (16, 8), (3, 2), (7, 3), (16, 2)]


@pytest.mark.parametrize("L_high,L_low", LEVELS)
def test_levels_quantize_and_decode(L_high, L_low):
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=2, Lyr=2, H=2, H_q=8, T=333)
    k, v = synth.kv(wl, L_high * 17 + L_low, DEV)
    score = synth.uniform_score(wl, L_high, DEV)
    seq_len = torch.tensor([333, 201], dtype=torch.int32, device=DEV)
    r_ppm = 250_000 if L_high != L_low else 500_000
    cache, mask = _prefill(k, v, score, seq_len, L_high, L_low, r_ppm, wl.H_q)
    masks = _oracle_masks(score, [333, 201], r_ppm)
    m = to_np(mask)
    for b, T in enumerate([333, 201]):
        assert np.array_equal(m[b, :T], masks[b]) and not m[b, T:].any()
    assert _status(cache) == 0
    kn, vn = to_np(k), to_np(v)
    compare_pools(cache, kn, vn, masks, [333, 201], L_high, L_low)
    q = synth.decode_query(wl, 3, DEV)
    out = torch.empty_like(q)
    kv.semkv_decode_attn(cache, 0, 2, q, out)
    ref = _oracle_decode_slabs(kn, vn, masks, [333, 201], to_np(q), L_high, L_low)
    check_attention(to_np(out), ref)


# query heads per KV head: 1..3 leave MMA columns unused, 4 packs the low f16
# part of P' into the free columns, 6 and 8 use every column
@pytest.mark.parametrize("H,H_q", [(2, 2), (2, 4), (1, 3), (2, 8), (2, 12), (1, 8)])
def test_decode_gqa_group_sizes(H, H_q):
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=2, Lyr=2, H=H, H_q=H_q, T=333)
    k, v = synth.kv(wl, 40 + H_q, DEV)
    score = synth.uniform_score(wl, H_q, DEV)
    seq_len = torch.tensor([333, 201], dtype=torch.int32, device=DEV)
    cache, mask = _prefill(k, v, score, seq_len, 6, 5, 500_000, wl.H_q)
    masks = _oracle_masks(score, [333, 201], 500_000)
    assert _status(cache) == 0
    kn, vn = to_np(k), to_np(v)
    q = synth.decode_query(wl, 5, DEV)
    out = torch.empty_like(q)
    kv.semkv_decode_attn(cache, 0, 2, q, out)
    ref = _oracle_decode_slabs(kn, vn, masks, [333, 201], to_np(q), 6, 5)
    check_attention(to_np(out), ref)


# ----------------------------------------------------------------- adversarial rows
def _adversarial_rows(rng, n):
    rows = []
    for i in range(n):
        kind = i % 10
        if kind == 0:
            x = np.full(128, rng.standard_normal())                      # constant row
        elif kind == 1:
            x = np.where(rng.random(128) < 0.5, 0.0, -0.0)               # +-0 only
        elif kind == 2:
            x = rng.integers(0, 11, 128) * 0.5                           # half-integer ties (L=6: scale 1)
            x[0], x[1] = 0.0, 5.0
        elif kind == 3:
            x = rng.integers(0, 9, 128) * 0.625 / 2                      # ties for L=5 grid 1.25
            x[0], x[1] = 0.0, 5.0
        elif kind == 4:
            x = np.clip(rng.standard_normal(128) * 30000.0, -65504, 65504)   # near the fp16 range
            x[0] = 65504.0
            x[1] = -65504.0
        elif kind == 5:
            x = rng.standard_normal(128) * 1e-6                          # fp16 subnormals
        elif kind == 6:
            x = rng.standard_normal(128)
            x[rng.integers(128)] = 1000.0                                # one outlier
        elif kind == 7:
            x = np.full(128, 3.0)
            x[5] = 3.001                                                 # tiny range
        elif kind == 8:
            x = rng.integers(-3, 4, 128).astype(float)                   # few distinct values
        else:
            x = np.clip(rng.standard_normal(128) * rng.lognormal(0, 2), -65504, 65504)
        rows.append(x)
    return np.array(rows).astype(np.float16)


@pytest.mark.parametrize("L_high,L_low", [(6, 5), (3, 2), (16, 8), (5, 4)])
def test_adversarial_rows_bit_exact(L_high, L_low):
    kv = kv_mod()
    rng = np.random.default_rng(L_high)
    T = 200
    k = _adversarial_rows(rng, 2 * T).reshape(1, 1, 2, T, 128)
    v = _adversarial_rows(rng, 2 * T)[::-1].copy().reshape(1, 1, 2, T, 128)
    kt, vt = torch.from_numpy(k).to(DEV), torch.from_numpy(v).to(DEV)
    score = torch.from_numpy(rng.integers(0, 5, (1, T)).astype(np.float32)).to(DEV)   # heavy ties
    seq_len = torch.tensor([T], dtype=torch.int32, device=DEV)
    cache, mask = _prefill(kt, vt, score, seq_len, L_high, L_low, 500_000, 4)
    masks = _oracle_masks(score, [T], 500_000)
    assert np.array_equal(to_np(mask)[0], masks[0])
    assert _status(cache) == 0
    compare_pools(cache, k, v, masks, [T], L_high, L_low)


def test_nonfinite_rows_are_flagged():
    kv = kv_mod()
    rng = np.random.default_rng(5)
    k = rng.standard_normal((1, 1, 1, 64, 128)).astype(np.float16)
    v = rng.standard_normal((1, 1, 1, 64, 128)).astype(np.float16)
    k[0, 0, 0, 10, 3] = np.inf
    v[0, 0, 0, 20, 7] = np.nan
    score = torch.rand((1, 64), device=DEV)
    seq_len = torch.tensor([64], dtype=torch.int32, device=DEV)
    cache, mask = _prefill(torch.from_numpy(k).to(DEV), torch.from_numpy(v).to(DEV), score, seq_len, 6, 5,
                           500_000, 4)
    assert _status(cache) & kv.FLAG_NONFINITE
    # the finite rows are still exact
    masks = _oracle_masks(score, [64], 500_000)
    ok = np.ones(64, bool)
    ok[[10, 20]] = False
    for x, hw, lw, hm, lm in ((k, cache.k_high, cache.k_low, cache.k_high_meta, cache.k_low_meta),
                              (v, cache.v_high, cache.v_low, cache.v_high_meta, cache.v_low_meta)):
        ph, pl, _ = O.quantize_slab(x[0, 0, 0], masks[0], 6, 5)
        for cls, pool, words in ((1, ph, hw), (0, pl, lw)):
            toks = np.nonzero(masks[0] == cls)[0]
            sel = ok[toks]
            g = to_np(words[0, 0, 0, :len(toks)]).view(np.uint32)
            assert np.array_equal(g[sel], pool.words[sel])


def test_capacity_overflow_is_flagged_and_clamped():
    kv = kv_mod()
    rng = np.random.default_rng(6)
    T = 100
    k = torch.from_numpy(rng.standard_normal((1, 1, 1, T, 128)).astype(np.float16)).to(DEV)
    score = torch.rand((1, T), device=DEV)
    seq_len = torch.tensor([T], dtype=torch.int32, device=DEV)
    mask = torch.zeros((1, T), dtype=torch.uint8, device=DEV)
    kv.semkv_select(score, seq_len, 500_000, mask)
    cache = kv.MixedCache(1, 1, 1, 4, 6, 5, 500_000, 16, 16)
    kv.semkv_quantize(cache, k, k, seq_len, mask)
    assert _status(cache) & kv.FLAG_CAPACITY
    assert to_np(cache.n_high).tolist() == [16] and to_np(cache.n_low).tolist() == [16]
    masks = _oracle_masks(score, [T], 500_000)
    ph, pl, _ = O.quantize_slab(to_np(k)[0, 0, 0], masks[0], 6, 5)
    assert np.array_equal(to_np(cache.k_high[0, 0, 0]).view(np.uint32), ph.words[:16])
    assert np.array_equal(to_np(cache.k_low[0, 0, 0]).view(np.uint32), pl.words[:16])


# ----------------------------------------------------------------- select
@pytest.mark.parametrize("T", [1, 7, 128, 1000, 4099, 49152, 49153, 131072])
def test_select_bit_exact_with_ties(T):
    kv = kv_mod()
    rng = np.random.default_rng(T)
    B = 3
    lens = [T, max(1, T // 2), max(1, T - 3)]
    vals = np.array([0.0, -0.0, 1.5, -2.0, 3.25, 1e-38, -1e-38, 7.0], dtype=np.float32)
    s = np.where(rng.random((B, T)) < 0.5, rng.choice(vals, (B, T)), rng.standard_normal((B, T))).astype(np.float32)
    s[1] = rng.choice(vals[:3], T)                                   # almost all ties
    st = torch.from_numpy(s).to(DEV)
    seq_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
    for r_ppm in (0, 1, 100_000, 333_333, 500_000, 900_000, 999_999, 1_000_000):
        mask = torch.full((B, T), 7, dtype=torch.uint8, device=DEV)
        kv.semkv_select(st, seq_len, r_ppm, mask)
        m = to_np(mask)
        for b in range(B):
            ref = O.select_mask(s[b, :lens[b]], O.num_high(lens[b], r_ppm))
            assert np.array_equal(m[b, :lens[b]], ref), (b, r_ppm)
            assert not m[b, lens[b]:].any()


def test_select_nan_flag():
    kv = kv_mod()
    s = torch.rand((1, 100), device=DEV)
    s[0, 50] = float("nan")
    mask = torch.zeros((1, 100), dtype=torch.uint8, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    kv.semkv_select(s, torch.tensor([100], dtype=torch.int32, device=DEV), 500_000, mask, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & kv.FLAG_NONFINITE


# ----------------------------------------------------------------- scores
@pytest.mark.parametrize("kdist", ["lognormal", "x10ch"])
def test_key_l2_bit_exact(kdist):
    kv = kv_mod()
    wl = synth.scaled(synth.MISTRAL_LONG, Lyr=2, T=3000, B=2, kdist=kdist)
    k, _ = synth.kv(wl, 9, DEV)
    seq_len = torch.tensor([3000, 1234], dtype=torch.int32, device=DEV)
    score = torch.full((2, 3000), -1.0, device=DEV)
    layer = 1
    kl = k[:, layer]
    kv.semkv_score(kv.SCORE_KEY_L2, kl, k.stride(0), None, seq_len, 2, 3000, 8, 32, 64, score)
    s = to_np(score)
    kn = to_np(k)
    for b, T in enumerate([3000, 1234]):
        ref = O.score_key_l2(kn[b, layer, :, :T])
        assert np.array_equal(s[b, :T].view(np.uint32), ref.view(np.uint32))
        assert not s[b, T:].any()


# window groups of 256 rows (the shipped shape), 64 and 129 (padded row tiles,
# sequences shorter than the window) and 512 rows (wider than one tensor-memory
# accumulator: the mma.sync path)
@pytest.mark.parametrize("H,H_q,w,lens", [(2, 8, 64, [700, 50]), (8, 32, 64, [2048, 1500]), (1, 4, 16, [333, 5]),
                                          (2, 6, 43, [517, 40]), (1, 8, 64, [1000, 64])])
def test_attn_mass_within_tolerance(H, H_q, w, lens):
    kv = kv_mod()
    T = max(lens)
    wl = synth.scaled(synth.LLAMA_PREFILL, B=len(lens), Lyr=1, H=H, H_q=H_q, T=T, w=w)
    k, _ = synth.kv(wl, 11, DEV)
    q = synth.q_window(wl, 11, DEV)
    seq_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
    score = torch.full((len(lens), T), -1.0, device=DEV)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, 0], k.stride(0), q, seq_len, len(lens), T, H, H_q, w, score)
    s = to_np(score)
    kn, qn = to_np(k), to_np(q)
    for b, Tb in enumerate(lens):
        ref = O.score_attn_mass(kn[b, 0], qn[b], Tb)
        assert np.all(np.abs(s[b, :Tb] - ref) <= SCORE_RTOL * np.abs(ref) + SCORE_ATOL), b
        assert not s[b, Tb:].any()
        # ranking: the GPU mask (from GPU scores) agrees with the oracle's mask
        # (from oracle scores) except at tokens within the tolerance of the threshold
        mask = torch.zeros((1, T), dtype=torch.uint8, device=DEV)
        kv.semkv_select(score[b:b + 1].clone(), seq_len[b:b + 1].clone(), 500_000, mask)
        nh = O.num_high(Tb, 500_000)
        check_mask_near_threshold(to_np(mask)[0, :Tb], ref, O.select_mask(ref.astype(np.float32), nh), nh)


def test_attn_mass_deterministic():
    kv = kv_mod()
    wl = synth.scaled(synth.LLAMA_PREFILL, B=1, Lyr=1, T=4096)
    k, _ = synth.kv(wl, 12, DEV)
    q = synth.q_window(wl, 12, DEV)
    seq_len = torch.tensor([4096], dtype=torch.int32, device=DEV)
    outs = []
    for _ in range(2):
        score = torch.empty((1, 4096), device=DEV)
        kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, 0], k.stride(0), q, seq_len, 1, 4096, 8, 32, 64, score)
        outs.append(to_np(score))
    assert np.array_equal(outs[0].view(np.uint32), outs[1].view(np.uint32))


# ----------------------------------------------------------------- generation (block-exact)
@pytest.mark.parametrize("block,chunk", [(128, 1), (128, 50), (16, 3)])
def test_generation_block_exact(block, chunk):
    kv = kv_mod()
    rng = np.random.default_rng(block + chunk)
    B, Lyr, H, H_q = 3, 2, 2, 8
    lens = [300, 517, 128]
    T = max(lens)
    L_high, L_low, r_ppm = 6, 5, 500_000
    k = rng.standard_normal((B, Lyr, H, T, 128)).astype(np.float16)
    v = rng.standard_normal((B, Lyr, H, T, 128)).astype(np.float16)
    sc = rng.random((B, T)).astype(np.float32)
    steps = 300
    cache, mask = _prefill(torch.from_numpy(k).to(DEV), torch.from_numpy(v).to(DEV), torch.from_numpy(sc).to(DEV),
                           torch.tensor(lens, dtype=torch.int32, device=DEV), L_high, L_low, r_ppm, H_q,
                           block=block, gen=steps)
    ref = O.MixedCache(B, Lyr, H, L_high, L_low, r_ppm, block=block)
    ref.prefill(k, v, lens, _oracle_masks(torch.from_numpy(sc), lens, r_ppm))
    done = 0
    while done < steps:
        n = min(chunk, steps - done)
        kn = rng.standard_normal((B, Lyr, H, n, 128)).astype(np.float16)
        vn = rng.standard_normal((B, Lyr, H, n, 128)).astype(np.float16)
        sn = rng.random((B, n)).astype(np.float32)
        sn[:, ::7] = 0.5                                              # ties inside blocks
        kv.semkv_append_block(cache, torch.from_numpy(kn).to(DEV), torch.from_numpy(vn).to(DEV),
                              torch.from_numpy(sn).to(DEV), n)
        ref.append(kn, vn, sn)
        done += n
        assert cache.buf_len == ref.buf_k.shape[3] < block
        if done % 97 < chunk or done == steps:
            q = rng.standard_normal((B, Lyr, H_q, 128)).astype(np.float16)
            out = torch.empty((B, Lyr, H_q, 128), dtype=torch.float16, device=DEV)
            kv.semkv_decode_attn(cache, 0, Lyr, torch.from_numpy(q).to(DEV), out)
            check_attention(to_np(out), ref.decode(q))
    assert to_np(cache.n_high).tolist() == ref.n_high.tolist()
    assert to_np(cache.n_low).tolist() == ref.n_low.tolist()
    kv.semkv_append_block(cache, None, None, None, 0, kv.FLUSH)
    ref.flush()
    assert cache.buf_len == 0
    assert to_np(cache.n_high).tolist() == ref.n_high.tolist()
    assert _status(cache) == 0
    # every pool row equals the oracle's
    for b in range(B):
        for l in range(Lyr):
            for h in range(H):
                for which, words, meta in (("kh", cache.k_high, cache.k_high_meta), ("kl", cache.k_low, cache.k_low_meta),
                                           ("vh", cache.v_high, cache.v_high_meta), ("vl", cache.v_low, cache.v_low_meta)):
                    p = ref.pools(b, l, h, which)
                    n = p.words.shape[0]
                    if n == 0:
                        continue
                    assert np.array_equal(to_np(words[b, l, h, :n]).view(np.uint32), p.words)
                    gm = to_np(meta[b, l, h, :n])
                    assert np.array_equal(gm[:, 0], p.mn) and np.array_equal(gm[:, 1], p.scale)
    q = rng.standard_normal((B, Lyr, H_q, 128)).astype(np.float16)
    out = torch.empty((B, Lyr, H_q, 128), dtype=torch.float16, device=DEV)
    kv.semkv_decode_attn(cache, 0, Lyr, torch.from_numpy(q).to(DEV), out)
    check_attention(to_np(out), ref.decode(q))


@pytest.mark.parametrize("block,rotate", [(16, False), (128, False), (16, True)])
def test_generation_attention_mass_accumulation(block, rotate):
    """Scores of generated tokens from the attention they receive at the scoring
    layer: buf_score matches the oracle within the score tolerance after every
    step, and each block is ranked on the GPU's accumulated scores (the oracle
    takes the GPU score vector at the ranking, as for prefill), so every pool
    row stays bit-exact."""
    kv = kv_mod()
    rng = np.random.default_rng(90 + block)
    B, Lyr, H, H_q = 2, 2, 2, 8
    lens = [70, 45]
    T = max(lens)
    L_high, L_low, r_ppm = 6, 5, 500_000
    k = rng.standard_normal((B, Lyr, H, T, 128)).astype(np.float16)
    v = rng.standard_normal((B, Lyr, H, T, 128)).astype(np.float16)
    sc = rng.random((B, T)).astype(np.float32)
    steps = block + 9
    score_layer = Lyr - 1
    cache, _ = _prefill(torch.from_numpy(k).to(DEV), torch.from_numpy(v).to(DEV), torch.from_numpy(sc).to(DEV),
                        torch.tensor(lens, dtype=torch.int32, device=DEV), L_high, L_low, r_ppm, H_q,
                        block=block, gen=steps, rotate=rotate)
    ref = O.MixedCache(B, Lyr, H, L_high, L_low, r_ppm, block=block, rotate=rotate)
    ref.prefill(k, v, lens, _oracle_masks(torch.from_numpy(sc), lens, r_ppm))
    zeros = np.zeros((B, 1), np.float32)
    for step in range(steps):
        kn = rng.standard_normal((B, Lyr, H, 1, 128)).astype(np.float16)
        vn = rng.standard_normal((B, Lyr, H, 1, 128)).astype(np.float16)
        if ref.buf_k.shape[3] == block - 1:
            # this append completes the block: rank it on the GPU's scores
            ref.buf_score = to_np(cache.buf_score)[:, :block - 1].copy()
        kv.semkv_append_block(cache, torch.from_numpy(kn).to(DEV), torch.from_numpy(vn).to(DEV),
                              torch.from_numpy(zeros).to(DEV), 1)
        ref.append(kn, vn, zeros)
        q = rng.standard_normal((B, Lyr, H_q, 128)).astype(np.float16)
        out = torch.empty((B, Lyr, H_q, 128), dtype=torch.float16, device=DEV)
        kv.semkv_decode_attn_acc(cache, 0, Lyr, score_layer, torch.from_numpy(q).to(DEV), out)
        check_attention(to_np(out), ref.decode(q, score_layer=score_layer))
        nb = cache.buf_len
        assert nb == ref.buf_k.shape[3]
        gs = to_np(cache.buf_score)[:, :nb].astype(np.float64)
        rs = ref.buf_score.astype(np.float64)
        assert np.all(np.abs(gs - rs) <= SCORE_RTOL * np.abs(rs) + SCORE_ATOL), step
    assert _status(cache) == 0
    assert to_np(cache.n_high).tolist() == ref.n_high.tolist()
    for b in range(B):
        for l in range(Lyr):
            for h in range(H):
                for which, words in (("kh", cache.k_high), ("kl", cache.k_low), ("vh", cache.v_high),
                                     ("vl", cache.v_low)):
                    p = ref.pools(b, l, h, which)
                    n = p.words.shape[0]
                    assert np.array_equal(to_np(words[b, l, h, :n]).view(np.uint32), p.words)


def test_decode_attn_acc_is_deterministic_and_matches_plain_decode():
    kv = kv_mod()
    rng = np.random.default_rng(77)
    B, Lyr, H, H_q, T = 1, 2, 2, 8, 200
    k = torch.from_numpy(rng.standard_normal((B, Lyr, H, T, 128)).astype(np.float16)).to(DEV)
    sc = torch.from_numpy(rng.random((B, T)).astype(np.float32)).to(DEV)
    cache, _ = _prefill(k, k, sc, torch.tensor([T], dtype=torch.int32, device=DEV), 6, 5, 500_000, H_q, gen=64)
    kn = torch.from_numpy(rng.standard_normal((B, Lyr, H, 50, 128)).astype(np.float16)).to(DEV)
    kv.semkv_append_block(cache, kn, kn, torch.zeros((B, 50), device=DEV), 50)
    q = torch.from_numpy(rng.standard_normal((B, Lyr, H_q, 128)).astype(np.float16)).to(DEV)
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    kv.semkv_decode_attn(cache, 0, Lyr, q, o1)
    s0 = cache.buf_score.clone()
    kv.semkv_decode_attn_acc(cache, 0, Lyr, 0, q, o2)
    assert torch.equal(o1, o2)                                        # same outputs
    d1 = cache.buf_score - s0
    cache.buf_score.copy_(s0)
    kv.semkv_decode_attn_acc(cache, 0, Lyr, 0, q, o2)
    assert torch.equal(cache.buf_score - s0, d1)                      # bitwise deterministic
    assert float(d1[0, 50:].abs().max()) == 0.0                       # only the 50 block tokens
    with pytest.raises(kv.SemkvError):
        kv.semkv_decode_attn_acc(cache, 0, 1, 1, q[:, :1].contiguous(), o2[:, :1].contiguous())


# ----------------------------------------------------------------- Hadamard rotation (Table 2)
@pytest.mark.parametrize("L_high,L_low,kdist", [(6, 5, "x10ch"), (6, 5, "lognormal"), (8, 6, "x10ch"),
                                                (4, 4, "x10ch"), (16, 2, "lognormal")])
def test_rotated_quantize_bit_exact_and_decode(L_high, L_low, kdist):
    kv = kv_mod()
    wl = synth.scaled(synth.TINY, B=2, Lyr=2, H=2, H_q=8, T=333, kdist=kdist)
    k, v = synth.kv(wl, 300 + L_high, DEV)
    score = synth.uniform_score(wl, L_low, DEV)
    seq_len = torch.tensor([333, 201], dtype=torch.int32, device=DEV)
    cache, mask = _prefill(k, v, score, seq_len, L_high, L_low, 500_000, wl.H_q, rotate=True)
    masks = _oracle_masks(score, [333, 201], 500_000)
    assert _status(cache) == 0
    kn, vn = to_np(k), to_np(v)
    compare_pools(cache, kn, vn, masks, [333, 201], L_high, L_low, rotate=True)
    ref = O.MixedCache(2, 2, 2, L_high, L_low, 500_000, rotate=True)
    ref.prefill(kn, vn, [333, 201], masks)
    q = synth.decode_query(wl, 9, DEV)
    out = torch.empty_like(q)
    kv.semkv_decode_attn(cache, 0, 2, q, out)
    check_attention(to_np(out), ref.decode(to_np(q)))


def test_rotated_adversarial_rows_bit_exact():
    kv = kv_mod()
    rng = np.random.default_rng(404)
    rows = _adversarial_rows(rng, 160)
    x = rows.reshape(1, 1, 1, 160, 128)
    sc = torch.from_numpy(rng.random((1, 160)).astype(np.float32)).to(DEV)
    xt = torch.from_numpy(x).to(DEV)
    cache, mask = _prefill(xt, xt, sc, torch.tensor([160], dtype=torch.int32, device=DEV), 6, 5, 500_000, 4,
                           rotate=True)
    masks = _oracle_masks(sc, [160], 500_000)
    assert _status(cache) == 0
    compare_pools(cache, x, x, masks, [160], 6, 5, rotate=True)


def test_rotation_needs_at_most_four_query_heads_per_kv_head():
    kv = kv_mod()
    cache = new_cache(1, 1, 1, 8, 6, 5, 500_000, 64, rotate=True)
    q = torch.zeros((1, 1, 8, 128), dtype=torch.float16, device=DEV)
    with pytest.raises(kv.SemkvError):
        kv.semkv_decode_attn(cache, 0, 1, q, torch.empty_like(q))


def test_decode_layer_subset_and_empty_sequence():
    kv = kv_mod()
    rng = np.random.default_rng(21)
    B, Lyr, H, H_q, T = 2, 3, 2, 4, 90
    k = rng.standard_normal((B, Lyr, H, T, 128)).astype(np.float16)
    v = rng.standard_normal((B, Lyr, H, T, 128)).astype(np.float16)
    sc = rng.random((B, T)).astype(np.float32)
    lens = [90, 0]
    cache, _ = _prefill(torch.from_numpy(k).to(DEV), torch.from_numpy(v).to(DEV), torch.from_numpy(sc).to(DEV),
                        torch.tensor(lens, dtype=torch.int32, device=DEV), 6, 5, 500_000, H_q)
    q = rng.standard_normal((B, 2, H_q, 128)).astype(np.float16)
    out = torch.full((B, 2, H_q, 128), 9.0, dtype=torch.float16, device=DEV)
    kv.semkv_decode_attn(cache, 1, 2, torch.from_numpy(q).to(DEV), out)
    o = to_np(out)
    masks = _oracle_masks(torch.from_numpy(sc), lens, 500_000)
    ref = _oracle_decode_slabs(k[:1], v[:1], masks[:1], lens[:1], q[:1], 6, 5, layer0=1)
    check_attention(o[:1], ref)
    assert np.all(o[1] == 0)                                          # no cached token: zeros
