"""Shared pieces of the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare."""
import numpy as np
import torch

from oracle import semkv_oracle as O

# decode-attention tolerance on fp16 outputs (relative L2 over a call, max-abs)
REL_L2 = 1e-3
MAX_ABS = 5e-3
# attention-mass score tolerance (relative to each score, plus an absolute floor)
SCORE_RTOL = 1e-4
SCORE_ATOL = 1e-6


def kv_mod():
    import kv_cache_mixed_b200 as kv   # fails loudly if libsemkv.so is missing
    return kv


def to_np(t):
    return t.detach().cpu().numpy()


def new_cache(B, Lyr, H, H_q, L_high, L_low, r_ppm, T_cap, block=128, gen=0, rotate=False):
    kv = kv_mod()
    cap_h = O.num_high(T_cap, r_ppm) + O.num_high(block, r_ppm) * (gen // block + 2) + 16
    cap_l = T_cap + block * (gen // block + 2) + 16
    return kv.MixedCache(B, Lyr, H, H_q, L_high, L_low, r_ppm, cap_h, cap_l, block=block, rotate=rotate)


def compare_pools(cache, k, v, masks, seq_len, L_high, L_low, layers=None, heads=None, rotate=False):
    """Bit-exact comparison of every pool row of the given (layer, head) slabs."""
    B, Lyr, H = k.shape[0], k.shape[1], k.shape[2]
    layers = range(Lyr) if layers is None else layers
    heads = range(H) if heads is None else heads
    n_high = to_np(cache.n_high)
    n_low = to_np(cache.n_low)
    for b in range(B):
        T = int(seq_len[b])
        m = masks[b][:T]
        assert n_high[b] == int(m.sum()) and n_low[b] == T - int(m.sum())
        for l in layers:
            for h in heads:
                for x, (ph_w, pl_w, ph_m, pl_m) in (
                        (k, (cache.k_high, cache.k_low, cache.k_high_meta, cache.k_low_meta)),
                        (v, (cache.v_high, cache.v_low, cache.v_high_meta, cache.v_low_meta))):
                    xs = to_np(x[b, l, h, :T]) if isinstance(x, torch.Tensor) else x[b, l, h, :T]
                    ph, pl, _ = O.quantize_slab(xs, m, L_high, L_low, rotate)
                    for pool, words, meta, n in ((ph, ph_w, ph_m, n_high[b]), (pl, pl_w, pl_m, n_low[b])):
                        gw = to_np(words[b, l, h, :n]).view(np.uint32)
                        gm = to_np(meta[b, l, h, :n])
                        assert np.array_equal(gw, pool.words), (b, l, h)
                        assert np.array_equal(gm[:, 0].view(np.uint32), pool.mn.view(np.uint32)), (b, l, h)
                        assert np.array_equal(gm[:, 1].view(np.uint32), pool.scale.view(np.uint32)), (b, l, h)


def check_mask_near_threshold(mask_gpu, score_ref, mask_ref, n_high):
    """A GPU mask from the GPU's own (tolerance-level) scores may differ from the
    oracle's mask only at tokens whose oracle score lies within the score
    tolerance of the oracle's threshold score; it keeps exactly n_high ones."""
    assert int(mask_gpu.sum()) == n_high
    diff = np.nonzero(mask_gpu != mask_ref)[0]
    if diff.size == 0:
        return 0
    order = np.lexsort((np.arange(score_ref.shape[0]), -score_ref))
    thr = score_ref[order[n_high - 1]] if n_high > 0 else np.inf
    band = SCORE_RTOL * abs(thr) * 2 + SCORE_ATOL * 2
    assert np.all(np.abs(score_ref[diff] - thr) <= band), (diff, score_ref[diff], thr)
    return int(diff.size)


def check_attention(out_gpu, out_ref):
    o = out_gpu.astype(np.float64)
    rel = np.linalg.norm(o - out_ref) / max(np.linalg.norm(out_ref), 1e-30)
    mx = np.max(np.abs(o - out_ref))
    print(f"[attention error] rel-L2 {rel:.3e} max-abs {mx:.3e}")
    assert rel <= REL_L2 and mx <= MAX_ABS, (rel, mx)
    return rel, mx
