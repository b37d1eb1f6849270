"""Seeded synthetic workloads shaped like the KV caches of the pages' backbones.

The backbones of SemKV (Table 2: Llama-3.1-8B-Instruct, Mistral-7B-Instruct-v0.3)
share one KV shape: 32 layers, 8 KV heads, 32 query heads, head_dim 128.  The
pages evaluate on LongBench and MT-Eval; no dataset is used here: these
generators stand in for them with seeded random tensors of the same shapes.

Every draw comes from a ``torch.Generator`` seeded from (seed, tensor id), on the
device the caller asks for, so a GPU test can draw full-size inputs on the GPU
and copy any slice to the host for the oracle.  Nothing here computes any part of
the method.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

D = 128

# tensor ids: each tensor of a workload draws from its own stream
_T_K, _T_V, _T_KSCALE, _T_KCH, _T_QWIN, _T_Q, _T_SCORE, _T_LEN, _T_NEWK, _T_NEWV, _T_NEWQ, _T_NEWS = range(12)


def gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + tensor_id * 7919) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


@dataclass(frozen=True)
class Workload:
    """Shapes and input distributions of one workload."""
    name: str
    B: int
    Lyr: int
    H: int
    H_q: int
    T: int                  # T_max (every sequence has T tokens unless lengths are drawn)
    kdist: str              # "x10ch": N(0,1) with 4 key channels x10; "lognormal": N(0,1) * exp(N(0,1)) per channel
    score: str              # "uniform" (given), "attn_mass", "key_l2"
    r_ppm: int
    L_high: int
    L_low: int
    w: int = 64
    len_lo: int = 0         # >0: per-sequence prompt lengths ~ U[len_lo, len_hi]
    len_hi: int = 0
    gen_steps: int = 0      # generation steps (new tokens per sequence)


# The five workloads.  Sizes are the full ones; tests shrink them where stated.
TINY = Workload("tiny", B=1, Lyr=1, H=1, H_q=4, T=256, kdist="x10ch", score="uniform",
                r_ppm=500_000, L_high=6, L_low=5)
LLAMA_PREFILL = Workload("llama8b_prefill_T32768", B=1, Lyr=32, H=8, H_q=32, T=32768,
                         kdist="lognormal", score="attn_mass", r_ppm=500_000, L_high=6, L_low=5)
GENERATION = Workload("llama8b_generation_B16", B=16, Lyr=32, H=8, H_q=32, T=16384,
                      kdist="lognormal", score="attn_mass", r_ppm=500_000, L_high=6, L_low=5,
                      len_lo=4096, len_hi=16384, gen_steps=512)
MISTRAL_LONG = Workload("mistral7b_T131072", B=1, Lyr=32, H=8, H_q=32, T=131072,
                        kdist="x10ch", score="key_l2", r_ppm=500_000, L_high=6, L_low=5)
LEVEL_SWEEP = Workload("level_sweep_B8_T32768", B=8, Lyr=1, H=8, H_q=32, T=32768,
                       kdist="x10ch", score="attn_mass", r_ppm=500_000, L_high=6, L_low=5)

WORKLOADS = {1: TINY, 2: LLAMA_PREFILL, 3: GENERATION, 4: MISTRAL_LONG, 5: LEVEL_SWEEP}
R_SWEEP_PPM = (100_000, 250_000, 500_000, 750_000, 900_000)
LEVEL_PAIRS = ((4, 4), (5, 5), (6, 6), (8, 8), (16, 16), (5, 4), (6, 5), (8, 6), (16, 8))


def seq_lens(wl: Workload, seed: int) -> torch.Tensor:
    """int32 [B] prompt lengths: U[len_lo, len_hi] when drawn, else all T."""
    if wl.len_lo > 0:
        g = gen(seed, _T_LEN, "cpu")
        return torch.randint(wl.len_lo, wl.len_hi + 1, (wl.B,), generator=g, dtype=torch.int64).to(torch.int32)
    return torch.full((wl.B,), wl.T, dtype=torch.int32)


def kv(wl: Workload, seed: int, device, layers=None):
    """K, V float16 [B][n_layers][H][T][D] for the given layers (default: all)."""
    layers = list(range(wl.Lyr)) if layers is None else list(layers)
    B, H, T = wl.B, wl.H, wl.T
    k = torch.empty((B, len(layers), H, T, D), dtype=torch.float16, device=device)
    v = torch.empty_like(k)
    # per-(layer, head, channel) key factors are drawn for all layers at once so
    # that any subset of layers sees the same factors
    if wl.kdist == "lognormal":
        fac = torch.exp(torch.randn((wl.Lyr, H, D), generator=gen(seed, _T_KSCALE, device), device=device))
    else:
        fac = torch.ones((wl.Lyr, H, D), device=device)
        g = gen(seed, _T_KCH, device)
        for l in range(wl.Lyr):
            for h in range(H):
                ch = torch.randperm(D, generator=g, device=device)[:4]
                fac[l, h, ch] = 10.0
    for i, l in enumerate(layers):
        gk = gen(seed, _T_K * 1000 + l, device)
        gv = gen(seed, _T_V * 1000 + l, device)
        for b in range(B):
            kk = torch.randn((H, T, D), generator=gk, device=device) * fac[l][:, None, :]
            k[b, i] = kk.to(torch.float16)
            v[b, i] = torch.randn((H, T, D), generator=gv, device=device).to(torch.float16)
    return k, v


def q_window(wl: Workload, seed: int, device) -> torch.Tensor:
    """float16 [B][H_q][w][D], the last w query rows of the scoring layer, ~N(0,1)."""
    g = gen(seed, _T_QWIN, device)
    return torch.randn((wl.B, wl.H_q, wl.w, D), generator=g, device=device).to(torch.float16)


def decode_query(wl: Workload, seed: int, device, step: int = 0, n_layers=None) -> torch.Tensor:
    """float16 [B][n_layers][H_q][D] decode queries ~N(0,1)."""
    nl = wl.Lyr if n_layers is None else n_layers
    g = gen(seed, _T_Q * 1000 + step, device)
    return torch.randn((wl.B, nl, wl.H_q, D), generator=g, device=device).to(torch.float16)


def uniform_score(wl: Workload, seed: int, device) -> torch.Tensor:
    """float32 [B][T] importance scores ~U(0,1), given directly."""
    g = gen(seed, _T_SCORE, device)
    return torch.rand((wl.B, wl.T), generator=g, device=device)


def new_tokens(wl: Workload, seed: int, step: int, device, n: int = 1):
    """Generated tokens: k, v float16 [B][Lyr][H][n][D] ~N(0,1); q float16 [B][Lyr][H_q][D]."""
    gk = gen(seed, _T_NEWK * 100_000 + step, device)
    gv = gen(seed, _T_NEWV * 100_000 + step, device)
    gq = gen(seed, _T_NEWQ * 100_000 + step, device)
    shape = (wl.B, wl.Lyr, wl.H, n, D)
    k = torch.randn(shape, generator=gk, device=device).to(torch.float16)
    v = torch.randn(shape, generator=gv, device=device).to(torch.float16)
    q = torch.randn((wl.B, wl.Lyr, wl.H_q, D), generator=gq, device=device).to(torch.float16)
    return k, v, q


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some sizes replaced (for oracle-sized tests)."""
    d = dict(wl.__dict__)
    d.update(kw)
    return Workload(**d)
