"""Benchmark of the SemKV hot path on one B200 (or N replicas, one per GPU).

One step = the whole hot path over one batch of the Llama-3.1-8B-shaped prefill
workload (32 layers, 8 KV heads, 32 query heads, head_dim 128, T = 32768,
batch 1, levels 6/5, r = 0.5; seeded synthetic fp16 K/V with a per-channel
lognormal key scale; the score is the attention mass from the last 64 query
rows of the last layer):
    a1 attention-mass score -> a2 top-r select -> a3/a4 quantize+pack of every
    K and V row -> a5 append one generated token -> a6 decode attention of one
    query per head over all 32 layers.
value = FP16 K+V input bytes of the batch / step time (GB/s).  Per-stage times,
quantize GB/s, decode GB/s and the roofline of the dominant kernel are
reported beside it.  Inputs (4 GiB) exceed L2 (126 MB), so no flush is needed.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With --gpus N > 1 (under torchrun) every rank runs an independent replica
(the path has no exchange step): scaling "weak", value = all ranks' bytes /
max-over-ranks time.  --impl reference times the CPU oracle on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# kernels one step launches: attention-mass score 4 (row stats, merge, column
# sums, head sum), select 1, quantize 3 (slot scan, quantize+pack, count
# advance), append 1, decode 4 (one pool kernel per level, FP16 block, merge)
LAUNCHES_PER_STEP = 4 + 1 + 3 + 1 + 4
METRIC = "KV quantize+pack GB/s (FP16 in) & mixed-prec decode-attn GB/s vs HBM roofline"
KERNEL_SOURCES = ["kv_cache_mixed_b200/csrc/quantize.cu", "kv_cache_mixed_b200/csrc/common.cuh"]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-options", action="store_true", help="skip the option timings (score accumulation, rotation)")
    ap.add_argument("--case", default=None, choices=["score", "select", "quantize", "decode"],
                    help="profiling case: run only this stage, on the prefill workload cut to --layers layers")
    ap.add_argument("--layers", type=int, default=4)
    return ap.parse_args(argv)


# ------------------------------------------------------------------ ranks
def init_ranks(backend="nccl", timeout_s=120):
    """(rank, world, torch.distributed or None) from the torchrun environment.
    Replicas only: the ranks exchange nothing on the data path, just a barrier
    around the timed region and a max-reduction of the step time."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world <= 1:
        return rank, world, None
    import datetime

    import torch
    import torch.distributed as tdist
    if backend == "nccl":
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world, tdist


def max_over_ranks(ms, dist, device):
    """The slowest rank's time (every rank takes this collective, in the same order)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world, bytes_per_rank, ms):
    """Whole-job GB/s: the bytes every rank processed over the slowest rank's time."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class Clocks:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, dist):
    import numpy as np
    import torch

    import kv_cache_mixed_b200 as kv
    from inputs import synth

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    dev = torch.device("cuda")
    wl = synth.LLAMA_PREFILL
    B, Lyr, H, H_q, T, w = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T, wl.w
    seed = 0
    k, v = synth.kv(wl, seed, dev)
    q_win = synth.q_window(wl, seed, dev)
    qdec = synth.decode_query(wl, seed, dev)
    kn, vn, _ = synth.new_tokens(wl, seed, 0, dev, n=1)
    sn = torch.rand((B, 1), device=dev)
    seq_len = synth.seq_lens(wl, seed).to(dev)
    score = torch.empty((B, T), device=dev)
    mask = torch.empty((B, T), dtype=torch.uint8, device=dev)
    out = torch.empty_like(qdec)
    cache = kv.MixedCache(B, Lyr, H, H_q, wl.L_high, wl.L_low, wl.r_ppm, kv.semkv_num_high(T, wl.r_ppm) + 128,
                          T - kv.semkv_num_high(T, wl.r_ppm) + 128)
    score_ws = torch.empty(max(1, int(kv.binding._lib_score_ws(0, B, T, H, H_q, w))), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    layer = Lyr - 1
    kl = k[:, layer]
    ev = {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for n in ("score", "select", "quantize", "append", "decode")}
    times = {n: [] for n in ev}

    def step(record):
        cache.n_high.zero_()
        cache.n_low.zero_()
        cache.c.buf_len = 0
        def mark(name, i):
            if record:
                ev[name][i].record(stream)
        mark("score", 0)
        kv.semkv_score(kv.SCORE_ATTN_MASS, kl, k.stride(0), q_win, seq_len, B, T, H, H_q, w, score, ws=score_ws)
        mark("score", 1)
        mark("select", 0)
        kv.semkv_select(score, seq_len, wl.r_ppm, mask)
        mark("select", 1)
        mark("quantize", 0)
        kv.semkv_quantize(cache, k, v, seq_len, mask)
        mark("quantize", 1)
        mark("append", 0)
        kv.semkv_append_block(cache, kn, vn, sn, 1)
        mark("append", 1)
        mark("decode", 0)
        kv.semkv_decode_attn(cache, 0, Lyr, qdec, out)
        mark("decode", 1)

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(torch.cuda.current_device()) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step(True)
            torch.cuda.synchronize()   # per-step stage events are read after each step
            for n, (a, b) in ev.items():
                times[n].append(a.elapsed_time(b))
        t1.record(stream)
        torch.cuda.synchronize()
    # the step loop above synchronizes per step for the stage events; the
    # headline is also timed without those syncs below
    # the clock sampler (one reading per 200 ms) starts with an untimed soak of
    # about 0.4 s of steps, so that it holds several readings under load next
    # to the short timed loop
    step_ms = max(statistics.median([sum(times[n][i] for n in times) for i in range(len(times["score"]))]), 1e-3)
    soak = int(400.0 / step_ms) + 1
    with Clocks(torch.cuda.current_device()) as clk2:
        for _ in range(soak):
            step(False)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t2, t3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t2.record(stream)
        for _ in range(args.steps):
            step(False)
        t3.record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
    ms = t2.elapsed_time(t3) / args.steps
    assert cache.status_flags() == 0, "device status flags set"
    ms = max_over_ranks(ms, dist, dev)

    # ---- algorithmic bytes
    nh = int(cache.n_high.sum().item())
    nl = int(cache.n_low.sum().item())
    Wh, Wl = kv.semkv_words_per_row(wl.L_high), kv.semkv_words_per_row(wl.L_low)
    fp16_in = 2 * B * Lyr * H * T * 128 * 2                      # K and V
    pool_bytes = 2 * Lyr * H * (nh * (4 * Wh + 8) + nl * (4 * Wl + 8))
    quant_bytes = fp16_in + pool_bytes + B * T * (1 + 4 + 4)      # + mask read, slot write+read
    # decode reads every pool row of K and V (codes + meta), the FP16 block and q, writes out
    dec_bytes = pool_bytes + 2 * B * Lyr * H * cache.buf_len * 256 + 2 * B * Lyr * H_q * 128 * 2
    stage = {n: statistics.median(v) for n, v in times.items()}
    q_ms = stage["quantize"]
    d_ms = stage["decode"]
    peak, peak_kind = peaks()
    achieved = quant_bytes / (q_ms * 1e-3) / 1e9
    traffic = None
    tp = os.path.join(ROOT, "profiles", "quantize_pack_traffic.json")
    if os.path.exists(tp):
        d = json.load(open(tp))
        import hashlib
        hsh = hashlib.sha256(b"".join(open(os.path.join(ROOT, f), "rb").read() for f in KERNEL_SOURCES)).hexdigest()
        if d.get("source_sha256") == hsh:
            traffic = d.get("dram_bytes_per_launch")
    value = job_value(world, fp16_in, ms)
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp16 in / fp32 quantize / mixed-radix u32 codes", "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "layers": Lyr, "kv_heads": H, "q_heads": H_q, "head_dim": 128,
                   "T": T, "L_high": wl.L_high, "L_low": wl.L_low, "r": wl.r_ppm / 1e6, "score": "attn_mass(w=64)",
                   "parallelism": "replicas" if world > 1 else "single-gpu",
                   "l2": "inputs 4 GiB > 126 MB L2, no flush"},
        "components": {
            "score_ms": round(stage["score"], 4), "select_ms": round(stage["select"], 4),
            "quantize_ms": round(q_ms, 4), "append_ms": round(stage["append"], 4), "decode_ms": round(d_ms, 4),
            "quantize_gbs_fp16_in": round(fp16_in / (q_ms * 1e-3) / 1e9, 1),
            "quantize_gbs_algorithmic": round(achieved, 1),
            "decode_gbs_cache_read": round(dec_bytes / (d_ms * 1e-3) / 1e9, 1),
            "decode_frac_of_hbm": round(dec_bytes / (d_ms * 1e-3) / 1e9 / peak, 3),
            "tokens_per_s_prefill": round(B * T / (ms * 1e-3), 1),
            "pool_bytes": pool_bytes, "compression_vs_fp16": round(fp16_in / pool_bytes, 3)},
        "roofline": {"kernel": "quantize_pack_kernel (+ slot scan and count kernels of semkv_quantize)",
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 3), "traffic": traffic, "peak_source": peak_kind},
        "clocks": clk2.summary(),
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
    }
    return res, (k, v, q_win, qdec, kn, vn, sn, seq_len, score, mask, out, cache, score_ws, fp16_in)


def run_extensions(state, reps=5):
    """Device times of the two options next to the headline path, on the same
    workload: decode with attention-mass accumulation for the FP16 block at
    the scoring layer, and the Hadamard-rotated cache (quantize and decode)."""
    import torch

    import kv_cache_mixed_b200 as kv
    from inputs import synth
    k, v, q_win, qdec, kn, vn, sn, seq_len, score, mask, out, cache, score_ws, fp16_in = state
    wl = synth.LLAMA_PREFILL
    B, Lyr, H, H_q, T = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for _ in range(reps):
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    acc_ms = timed(lambda: kv.semkv_decode_attn_acc(cache, 0, Lyr, Lyr - 1, qdec, out))
    nh = kv.semkv_num_high(T, wl.r_ppm)
    rc = kv.MixedCache(B, Lyr, H, H_q, wl.L_high, wl.L_low, wl.r_ppm, nh + 128, T - nh + 128, rotate=True)

    def rq():
        rc.n_high.zero_()
        rc.n_low.zero_()
        kv.semkv_quantize(rc, k, v, seq_len, mask)
    rq_ms = timed(rq)
    rd_ms = timed(lambda: kv.semkv_decode_attn(rc, 0, Lyr, qdec, out))
    assert rc.status_flags() == 0 and cache.status_flags() == 0
    return {"decode_acc_ms": round(acc_ms, 4),
            "rotated": {"quantize_ms": round(rq_ms, 4), "decode_ms": round(rd_ms, 4),
                        "quantize_gbs_fp16_in": round(fp16_in / (rq_ms * 1e-3) / 1e9, 1)}}


def run_e2e(args, state, dist=None):
    """Same step through the C ABI with pinned HOST inputs: H2D copies of K, V,
    the query window, the decode query and the new token inside the timed
    region, and a D2H read of the decode output."""
    import torch

    import kv_cache_mixed_b200 as kv
    from inputs import synth
    k, v, q_win, qdec, kn, vn, sn, seq_len, score, mask, out, cache, score_ws, fp16_in = state
    wl = synth.LLAMA_PREFILL
    B, Lyr, H, H_q, T, w = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T, wl.w
    hk, hv = k.cpu().pin_memory(), v.cpu().pin_memory()
    hq, hqd, hkn, hvn, hsn = (t.cpu().pin_memory() for t in (q_win, qdec, kn, vn, sn))
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    stream = torch.cuda.current_stream()
    h2d = sum(t.numel() * t.element_size() for t in (hk, hv, hq, hqd, hkn, hvn, hsn))
    d2h = hout.numel() * hout.element_size()

    def step():
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        for d, h in ((q_win, hq), (qdec, hqd), (kn, hkn), (vn, hvn), (sn, hsn)):
            d.copy_(h, non_blocking=True)
        cache.n_high.zero_()
        cache.n_low.zero_()
        cache.c.buf_len = 0
        kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, Lyr - 1], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score,
                       ws=score_ws)
        kv.semkv_select(score, seq_len, wl.r_ppm, mask)
        kv.semkv_quantize(cache, k, v, seq_len, mask)
        kv.semkv_append_block(cache, kn, vn, sn, 1)
        kv.semkv_decode_attn(cache, 0, Lyr, qdec, out)
        hout.copy_(out, non_blocking=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    n = max(2, min(args.steps, 5))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    return {"value": round(fp16_in / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


# ------------------------------------------------------------------ CPU oracle
def oracle_step_sample(n_layers_sample=2):
    """Time the oracle on the same workload: the full score and select, and
    quantize+pack and decode for n_layers_sample of the 32 layers.  Returns
    (extrapolated seconds per full step, description)."""
    import numpy as np
    import torch

    from inputs import synth
    from oracle import semkv_oracle as O
    wl = synth.LLAMA_PREFILL
    layers = list(range(wl.Lyr - n_layers_sample, wl.Lyr))
    k, v = synth.kv(wl, 0, "cpu", layers=layers)
    q_win = synth.q_window(wl, 0, "cpu")
    qdec = synth.decode_query(wl, 0, "cpu")
    k, v, q_win, qdec = (t.numpy() for t in (k, v, q_win, qdec))
    T = wl.T
    t0 = time.perf_counter()
    s = O.score_attn_mass(k[0, -1], q_win[0], T).astype(np.float32)
    mask = O.select_mask(s, O.num_high(T, wl.r_ppm))
    t1 = time.perf_counter()
    cache = O.MixedCache(1, n_layers_sample, wl.H, wl.L_high, wl.L_low, wl.r_ppm)
    cache.prefill(k, v, [T], [mask])
    cache.decode(qdec[:, layers])
    t2 = time.perf_counter()
    per_step = (t1 - t0) + (t2 - t1) * wl.Lyr / n_layers_sample
    desc = (f"attention-mass score + select over all T={T}, quantize+pack and decode of {n_layers_sample} of "
            f"{wl.Lyr} layers (all heads, all tokens), extrapolated to {wl.Lyr} layers; measured "
            f"{t2 - t0:.1f} s")
    return per_step, desc


def oracle_threads():
    """Threads the oracle can use: numpy's BLAS pool (its only multi-threaded part)."""
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline_json():
    # 7 of 32 layers: about 10 s of host work on the GPU machine
    per_step, desc = oracle_step_sample(7)
    fp16_in = 2 * 32 * 8 * 32768 * 128 * 2
    return {"value": round(fp16_in / per_step / 1e9, 4), "unit": "GB/s", "cores": oracle_threads(),
            "kind": "oracle", "sample": desc}


def run_reference(args, rank):
    if rank != 0:
        return None
    import torch
    times = []
    desc = ""
    # each step is one bounded sample of the workload (1 of 32 layers, plus the
    # full score and select), extrapolated to the full step; one untimed warm-up
    if args.warmup > 0:
        oracle_step_sample(1)
    for i in range(args.steps):
        per_step, desc = oracle_step_sample(1)
        times.append(per_step)
    per_step = statistics.median(times)
    fp16_in = 2 * 32 * 8 * 32768 * 128 * 2
    value = fp16_in / per_step / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64 (numpy)",
            "data": "synthetic",
            "config": {"workload": "llama8b_prefill_T32768", "B": 1, "layers": 32, "kv_heads": 8, "q_heads": 32,
                       "head_dim": 128, "T": 32768, "L_high": 6, "L_low": 5, "r": 0.5},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": oracle_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_case(args):
    """One stage alone, repeated warmup+steps times, on the prefill workload cut
    to args.layers layers (for ncu captures of a single kernel on a small case)."""
    import torch

    import kv_cache_mixed_b200 as kv
    from inputs import synth
    dev = torch.device("cuda")
    wl = synth.scaled(synth.LLAMA_PREFILL, Lyr=args.layers)
    B, Lyr, H, H_q, T, w = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T, wl.w
    k, v = synth.kv(wl, 0, dev)
    q_win = synth.q_window(wl, 0, dev)
    qdec = synth.decode_query(wl, 0, dev)
    seq_len = synth.seq_lens(wl, 0).to(dev)
    score = torch.empty((B, T), device=dev)
    mask = torch.empty((B, T), dtype=torch.uint8, device=dev)
    out = torch.empty_like(qdec)
    nh = kv.semkv_num_high(T, wl.r_ppm)
    cache = kv.MixedCache(B, Lyr, H, H_q, wl.L_high, wl.L_low, wl.r_ppm, nh + 128, T - nh + 128)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, Lyr - 1], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    torch.cuda.synchronize()
    for _ in range(args.warmup + args.steps):
        if args.case == "score":
            kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, Lyr - 1], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
        elif args.case == "select":
            kv.semkv_select(score, seq_len, wl.r_ppm, mask)
        elif args.case == "quantize":
            cache.n_high.zero_()
            cache.n_low.zero_()
            kv.semkv_quantize(cache, k, v, seq_len, mask)
        else:
            kv.semkv_decode_attn(cache, 0, Lyr, qdec, out)
    torch.cuda.synchronize()
    assert cache.status_flags() == 0
    print(json.dumps({"case": args.case, "layers": Lyr, "ok": True}))


def main():
    args = parse()
    if args.case:
        run_case(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, dist = init_ranks("nccl")
    res, state = run_ours(args, rank, world, dist)
    if not args.no_options:
        res["options"] = run_extensions(state)
    if not args.no_e2e:
        e2e = run_e2e(args, state, dist)
        if dist:
            e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], dist, "cuda")
            e2e["value"] = round(job_value(world, state[-1], e2e["ms_per_step"]), 2)
        res["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline_json()
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
