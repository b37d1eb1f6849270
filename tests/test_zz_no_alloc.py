"""semkv_quantize_noalloc: the quantize entry point for callers that cannot
allocate device memory (an engine whose memory all belongs to its own pool
allocator, a plugin host that forbids cudaMalloc on its hot path).  It must
give exactly what semkv_quantize gives with a caller workspace, call after
call, although every call reuses the same fixed scratch array.

This file is named to be collected last, so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from inputs import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _pools(cache):
    torch.cuda.synchronize()
    return {name: getattr(cache, name).cpu().numpy().copy()
            for name in ("k_high", "v_high", "k_low", "v_low", "k_high_meta", "v_high_meta",
                         "k_low_meta", "v_low_meta", "n_high", "n_low", "status")}


def _call(kv, k, v, seq_len, mask, r_ppm, use_workspace):
    B, Lyr, H, T = k.shape[:4]
    nh = kv.semkv_num_high(T, r_ppm)
    cache = kv.MixedCache(B, Lyr, H, 8, 6, 5, r_ppm, nh + 32, T - nh + 32)
    if use_workspace:
        kv.semkv_quantize(cache, k, v, seq_len, mask)
    else:
        kv.semkv_quantize_noalloc(cache, k, v, seq_len, mask)
    return _pools(cache)


def test_noalloc_quantize_equals_workspace_quantize_on_two_calls_in_a_row():
    import kv_cache_mixed_b200 as kv
    # two different calls: the second one runs on whatever the first left in
    # the shared scratch array (longer sequences first, then shorter ones)
    for seed, lens in ((0, [700, 513, 64]), (1, [300, 1, 299])):
        wl = synth.scaled(synth.TINY, B=3, Lyr=2, H=2, H_q=8, T=700)
        k, v = synth.kv(wl, seed, DEV)
        seq_len = torch.tensor(lens, dtype=torch.int32, device=DEV)
        score = synth.uniform_score(wl, seed, DEV)
        mask = torch.zeros((3, 700), dtype=torch.uint8, device=DEV)
        kv.semkv_select(score, seq_len, 500_000, mask)
        ref = _call(kv, k, v, seq_len, mask, 500_000, use_workspace=True)
        got = _call(kv, k, v, seq_len, mask, 500_000, use_workspace=False)
        for name in ref:
            assert np.array_equal(ref[name].view(np.uint8), got[name].view(np.uint8)), (seed, name)
        assert int(got["status"][0]) == 0
        assert got["n_high"].tolist() == [kv.semkv_num_high(n, 500_000) for n in lens]


def test_noalloc_quantize_rejects_sizes_beyond_its_scratch():
    import kv_cache_mixed_b200 as kv
    B, T = 2, 600_000              # needs about 4.8 MB of scratch, more than the array holds
    k = torch.zeros((B, 1, 1, T, 128), dtype=torch.float16, device=DEV)
    seq_len = torch.tensor([T, T], dtype=torch.int32, device=DEV)
    mask = torch.zeros((B, T), dtype=torch.uint8, device=DEV)
    cache = kv.MixedCache(B, 1, 1, 4, 6, 5, 500_000, 16, 16)
    with pytest.raises(kv.SemkvError, match="ERR_WORKSPACE"):
        kv.semkv_quantize_noalloc(cache, k, k, seq_len, mask)
    torch.cuda.synchronize()
    assert cache.status_flags() == 0 and cache.n_high.sum().item() == 0   # nothing was enqueued
