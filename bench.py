"""Benchmark of the SemKV hot path on one B200 (or N replicas, one per GPU).

Default workload (one JSON line, the headline): the Llama-3.1-8B-shaped prefill
cache (32 layers, 8 KV heads, 32 query heads, head_dim 128, T = 32768, batch 1,
levels 6/5, r = 0.5; seeded synthetic fp16 K/V with a per-channel lognormal key
scale; the score is the attention mass from the last 64 query rows of the last
layer).  One step is the whole hot path over that batch:
    a1 attention-mass score -> a2 top-r select -> a3/a4 quantize+pack of every
    K and V row -> a5 append one generated token -> a6 decode attention of one
    query per head over all 32 layers.
value = FP16 K+V input bytes of the batch / step time (GB/s).  Per-stage times,
quantize GB/s, decode GB/s and the rooflines of both kernels are reported
beside it.  Inputs (4 GiB) exceed L2 (126 MB), so no flush is needed.

Other workloads, one JSON line each (--workload):
    llama8b_generation_B16   batch 16, prompts ~U[4096, 16384], 512 generated
                             tokens through the FP16 block (key-L2 score of each
                             new token), decode of all 32 layers every step:
                             value = decode GB/s (pools + FP16 block read),
                             tokens/s and block-flush time beside it;
    mistral7b_T131072        T = 131072, key-L2 score, r swept over
                             {0.1, 0.25, 0.5, 0.75, 0.9}: quantize and decode
                             (64 steps) GB/s per r; value = quantize GB/s at r = 0.5;
    level_sweep_B8_T32768    batch 8, one layer, attention-mass score, uniform
                             L in {4,5,6,8,16} and pairs 5/4, 6/5, 8/6, 16/8:
                             quantize and decode GB/s per level; value =
                             quantize GB/s at 6/5.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

With --gpus N > 1 (under torchrun) every rank runs an independent replica
(the path has no exchange step): scaling "weak", value = all ranks' bytes /
max-over-ranks time.  --impl reference times the CPU oracle on a bounded
sample of the default workload.
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

# kernels one default step launches: attention-mass score 4 (pass 1, merge,
# pass 2, head sum), select 1, quantize 2 (slot scan with the count advance,
# quantize+pack), append 1, decode 3 (both pools in one launch -- every level
# pair the workloads use has a merged instance --, FP16 block, merge)
LAUNCHES_PER_STEP = 4 + 1 + 2 + 1 + 3
DECODE_LAUNCHES = 3
QUANT_LAUNCHES = 2
METRIC = "KV quantize+pack GB/s (FP16 in) & mixed-prec decode-attn GB/s vs HBM roofline"
KERNEL_SOURCES = ["kv_cache_mixed_b200/csrc/quantize.cu", "kv_cache_mixed_b200/csrc/common.cuh"]
DECODE_SOURCES = ["kv_cache_mixed_b200/csrc/decode.cu", "kv_cache_mixed_b200/csrc/common.cuh"]
NOMINAL_HBM_GBS = 8000.0          # the 8 TB/s HBM3e figure the throughput target is stated against
DEFAULT_WORKLOAD = "llama8b_prefill_T32768"
WORKLOAD_NAMES = [DEFAULT_WORKLOAD, "llama8b_generation_B16", "mistral7b_T131072", "level_sweep_B8_T32768"]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=WORKLOAD_NAMES)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-options", action="store_true", help="skip the option timings (score accumulation, rotation)")
    ap.add_argument("--case", default=None, choices=["score", "select", "quantize", "decode", "quantize_rotated",
                                                     "quantize_pages"],
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
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    return 6650.0, "fallback (6.65 TB/s, an earlier copy measurement on this pool)"


def roofline(kernel, algo_bytes, ms, traffic=None):
    """HBM roofline of one kernel: algorithmic bytes per launch over its event time."""
    peak, src = peaks()
    achieved = algo_bytes / (ms * 1e-3) / 1e9
    return {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 3), "frac_vs_8TBs": round(achieved / NOMINAL_HBM_GBS, 3),
            "bytes_per_launch": int(algo_bytes), "ms_per_launch": round(ms, 4), "traffic": traffic,
            "peak_source": src}


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


def event_times(fn, warmup, reps, stream):
    """Device times (ms) of `reps` calls of fn, each bracketed by CUDA events on
    the launching stream, after `warmup` untimed calls."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return ts


def soak(fn, ms_each, seconds=0.4):
    """Untimed repetitions for about `seconds`, so the clock sampler sees the GPU under load."""
    for _ in range(int(seconds * 1e3 / max(ms_each, 1e-3)) + 1):
        fn()


def pool_row_bytes(L):
    import kv_cache_mixed_b200 as kv
    return 4 * kv.semkv_words_per_row(L) + 8


def quant_algo_bytes(B, Lyr, H, T_tokens, nh_tokens, nl_tokens, Lh, Ll, T_stride):
    """quantize_pack: per row 256 B read + the pool row written; per token the
    mask byte read and the slot word written and read (K and V rows)."""
    return (2 * Lyr * H * (T_tokens * 256 + nh_tokens * pool_row_bytes(Lh) + nl_tokens * pool_row_bytes(Ll))
            + B * T_stride * (1 + 4 + 4))


def decode_algo_bytes(Lyr, H, H_q, B, nh_tokens, nl_tokens, Lh, Ll, buf_len):
    """decode: every pool row of K and V (codes + meta), the FP16 block, q and out."""
    return (2 * Lyr * H * (nh_tokens * pool_row_bytes(Lh) + nl_tokens * pool_row_bytes(Ll))
            + 2 * B * Lyr * H * buf_len * 256 + 2 * B * Lyr * H_q * 128 * 2)


def measured_traffic(record="quantize_pack_traffic.json", sources=None):
    """Per-launch DRAM bytes of a kernel from its committed ncu capture record
    (profiles/<record>), if it was taken on the current kernel sources (else None)."""
    tp = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(tp):
        return None
    import hashlib
    d = json.load(open(tp))
    hsh = hashlib.sha256(b"".join(open(os.path.join(ROOT, f), "rb").read()
                                  for f in (sources or KERNEL_SOURCES))).hexdigest()
    return d.get("dram_bytes_per_launch") if d.get("source_sha256") == hsh else None


def measured_decode_traffic():
    return measured_traffic("decode_pool_traffic.json", DECODE_SOURCES)


def cpu_cores_used(fn):
    """Run fn on the host; returns (result, wall seconds, cores actually used =
    process CPU time / wall time, threads available)."""
    t0, c0 = time.perf_counter(), time.process_time()
    r = fn()
    wall, cpu = time.perf_counter() - t0, time.process_time() - c0
    return r, wall, round(cpu / max(wall, 1e-9), 2), os.cpu_count()


# ------------------------------------------------------------------ default workload
def run_prefill(args, rank, world, dist):
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
    # per-stage device times: events around each stage, read after each step
    for _ in range(args.steps):
        step(True)
        torch.cuda.synchronize()
        for n, (a, b) in ev.items():
            times[n].append(a.elapsed_time(b))
    # the headline: K steps back to back with no host sync inside, after an
    # untimed soak of about 0.4 s so that the clock sampler sees the GPU under load
    step_ms = max(statistics.median([sum(times[n][i] for n in times) for i in range(len(times["score"]))]), 1e-3)
    with Clocks(torch.cuda.current_device()) as clk:
        soak(lambda: step(False), step_ms)
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
    fp16_in = 2 * B * Lyr * H * T * 128 * 2                      # K and V
    pool_bytes = 2 * Lyr * H * (nh * pool_row_bytes(wl.L_high) + nl * pool_row_bytes(wl.L_low))
    quant_bytes = quant_algo_bytes(B, Lyr, H, B * T, nh, nl, wl.L_high, wl.L_low, T)
    dec_bytes = decode_algo_bytes(Lyr, H, H_q, B, nh, nl, wl.L_high, wl.L_low, cache.buf_len)
    stage = {n: statistics.median(v) for n, v in times.items()}
    q_ms, d_ms = stage["quantize"], stage["decode"]
    rq = roofline("quantize_pack_kernel (+ slot scan and count kernels of semkv_quantize)", quant_bytes, q_ms,
                  measured_traffic())
    rd = roofline("decode_pool_kernel (both pools) + decode_buffer_kernel + decode_merge_kernel (semkv_decode_attn)",
                  dec_bytes, d_ms, measured_decode_traffic())
    value = job_value(world, fp16_in, ms)
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp16 in / fp32 quantize / mixed-radix u32 codes", "data": "synthetic",
        "config": prefill_config(world),
        "components": {
            "score_ms": round(stage["score"], 4), "select_ms": round(stage["select"], 4),
            "quantize_ms": round(q_ms, 4), "append_ms": round(stage["append"], 4), "decode_ms": round(d_ms, 4),
            "quantize_gbs_fp16_in": round(fp16_in / (q_ms * 1e-3) / 1e9, 1),
            "quantize_gbs_algorithmic": rq["achieved"],
            "decode_gbs_cache_read": rd["achieved"],
            "decode_frac_of_hbm": rd["frac"], "decode_frac_vs_8TBs": rd["frac_vs_8TBs"],
            "tokens_per_s_prefill": round(B * T / (ms * 1e-3), 1),
            "pool_bytes": pool_bytes, "compression_vs_fp16": round(fp16_in / pool_bytes, 3)},
        "roofline": rq,
        "rooflines": {"quantize": rq, "decode": rd},
        "clocks": clk.summary(),
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
    }
    return res, (k, v, q_win, qdec, kn, vn, sn, seq_len, score, mask, out, cache, score_ws, fp16_in)


def prefill_config(world=1):
    from inputs import synth
    wl = synth.LLAMA_PREFILL
    return {"workload": wl.name, "B": wl.B, "layers": wl.Lyr, "kv_heads": wl.H, "q_heads": wl.H_q, "head_dim": 128,
            "T": wl.T, "L_high": wl.L_high, "L_low": wl.L_low, "r": wl.r_ppm / 1e6, "score": "attn_mass(w=64)",
            "parallelism": "replicas" if world > 1 else "single-gpu",
            "l2": "inputs 4 GiB > 126 MB L2, no flush"}


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
    med = lambda fn: statistics.median(event_times(fn, 2, reps, stream))  # noqa: E731
    acc_ms = med(lambda: kv.semkv_decode_attn_acc(cache, 0, Lyr, Lyr - 1, qdec, out))
    nh = kv.semkv_num_high(T, wl.r_ppm)
    rc = kv.MixedCache(B, Lyr, H, H_q, wl.L_high, wl.L_low, wl.r_ppm, nh + 128, T - nh + 128, rotate=True)

    def rq():
        rc.n_high.zero_()
        rc.n_low.zero_()
        kv.semkv_quantize(rc, k, v, seq_len, mask)
    rq_ms = med(rq)
    rd_ms = med(lambda: kv.semkv_decode_attn(rc, 0, Lyr, qdec, out))
    assert rc.status_flags() == 0 and cache.status_flags() == 0
    del rc
    # the pages' own storage layout (groups of <= 5 digits in whole bits, rows
    # back to back in one bit stream, fp16 scalars)
    pc = kv.MixedCache(B, Lyr, H, H_q, wl.L_high, wl.L_low, wl.r_ppm, nh + 128, T - nh + 128,
                       layout=kv.LAYOUT_PAGES)

    def pq():
        pc.n_high.zero_()
        pc.n_low.zero_()
        kv.semkv_quantize(pc, k, v, seq_len, mask)
    pq_ms = med(pq)
    pd_ms = med(lambda: kv.semkv_decode_attn(pc, 0, Lyr, qdec, out))
    assert pc.status_flags() == 0
    pbytes = pc.pool_bytes()
    return {"decode_acc_ms": round(acc_ms, 4),
            "rotated": {"quantize_ms": round(rq_ms, 4), "decode_ms": round(rd_ms, 4),
                        "quantize_gbs_fp16_in": round(fp16_in / (rq_ms * 1e-3) / 1e9, 1)},
            "pages_layout": {"quantize_ms": round(pq_ms, 4), "decode_ms": round(pd_ms, 4),
                             "quantize_gbs_fp16_in": round(fp16_in / (pq_ms * 1e-3) / 1e9, 1),
                             "decode_gbs_cache_read": round(pbytes / (pd_ms * 1e-3) / 1e9, 1),
                             "pool_bytes": pbytes, "compression_vs_fp16": round(fp16_in / pbytes, 3),
                             "row_bits_high_low": [pc.row_bits_high, pc.row_bits_low]}}


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


# ------------------------------------------------------------------ other workloads
def _base_line(args, world, wl_name, value, ms, config, clk, launches):
    return {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp16 in / fp32 quantize / mixed-radix u32 codes", "data": "synthetic",
            "config": dict(config, workload=wl_name, parallelism="replicas" if world > 1 else "single-gpu"),
            "clocks": clk.summary(), "gpu_launches": launches}


def run_generation(args, rank, world, dist):
    """Batch 16, prompts ~U[4096, 16384]: the prompt is scored (attention mass),
    ranked and quantized once; then 512 generation steps, each: key-L2 score of
    the new token at the scoring layer, append (a block of 128 is ranked and
    quantized when it fills), decode of all 32 layers.  Warm-up steps run on
    the same cache, whose counts are then reset to the prompt's."""
    import numpy as np
    import torch

    import kv_cache_mixed_b200 as kv
    from inputs import synth
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    dev = torch.device("cuda")
    wl = synth.GENERATION
    B, Lyr, H, H_q, T, w, G = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T, wl.w, wl.gen_steps
    stream = torch.cuda.current_stream()
    seq_len = synth.seq_lens(wl, 0).to(dev)
    k, v = synth.kv(wl, 0, dev)
    q_win = synth.q_window(wl, 0, dev)
    score = torch.empty((B, T), device=dev)
    mask = torch.empty((B, T), dtype=torch.uint8, device=dev)
    nh_max = kv.semkv_num_high(T, wl.r_ppm)
    blocks = G // 128 + 2
    cache = kv.MixedCache(B, Lyr, H, H_q, wl.L_high, wl.L_low, wl.r_ppm, nh_max + blocks * 64 + 16,
                          T - nh_max + blocks * 128 + 16)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, Lyr - 1], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    qms = statistics.median(event_times(lambda: (cache.n_high.zero_(), cache.n_low.zero_(),
                                                 kv.semkv_quantize(cache, k, v, seq_len, mask)), 1, 3, stream))
    torch.cuda.synchronize()
    nh0, nl0 = cache.n_high.clone(), cache.n_low.clone()
    prompt_tokens = int(seq_len.sum().item())
    del k, v
    torch.cuda.empty_cache()
    # per-step inputs, drawn up front (the timed loop only launches kernels)
    news = [synth.new_tokens(wl, 0, s, dev, n=1) for s in range(max(G, args.warmup))]
    ones = torch.ones(B, dtype=torch.int32, device=dev)
    sn = torch.empty((B, 1), device=dev)
    out = torch.empty((B, Lyr, H_q, 128), dtype=torch.float16, device=dev)

    def gen_step(s, ev=None):
        kn, vn, qn = news[s]
        if ev:
            ev[0].record(stream)
        kv.semkv_score(kv.SCORE_KEY_L2, kn[:, Lyr - 1], kn.stride(0), None, ones, B, 1, H, H_q, w, sn)
        kv.semkv_append_block(cache, kn, vn, sn, 1)
        if ev:
            ev[1].record(stream)
        kv.semkv_decode_attn(cache, 0, Lyr, qn, out)
        if ev:
            ev[2].record(stream)

    def reset():
        cache.n_high.copy_(nh0)
        cache.n_low.copy_(nl0)
        cache.c.buf_len = 0

    for s in range(args.warmup):
        gen_step(s)
    torch.cuda.synchronize()
    reset()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(G)]
    buf_lens, flush = [], []
    with Clocks(torch.cuda.current_device()) as clk:
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        for s in range(G):
            flush.append(cache.buf_len == 127)           # this step's append fills the block
            gen_step(s, evs[s])
            buf_lens.append(cache.buf_len)               # FP16 tokens the decode of step s reads
        torch.cuda.synchronize()
    assert cache.status_flags() == 0, "device status flags set"
    app = np.array([e[0].elapsed_time(e[1]) for e in evs])
    dec = np.array([e[1].elapsed_time(e[2]) for e in evs])
    tot_ms = evs[0][0].elapsed_time(evs[-1][2])
    tot_ms = max_over_ranks(tot_ms, dist, dev)
    # decode bytes per step from the counts: prompt pools + quantized blocks + FP16 block
    nh_tok, nl_tok = int(nh0.sum().item()), int(nl0.sum().item())
    dbytes = []
    hb = kv.semkv_num_high(128, wl.r_ppm)
    for s in range(G):
        nb = sum(flush[:s + 1])
        dbytes.append(decode_algo_bytes(Lyr, H, H_q, B, nh_tok + B * nb * hb, nl_tok + B * nb * (128 - hb),
                                        wl.L_high, wl.L_low, buf_lens[s]))
    dec_gbs = sum(dbytes) / (dec.sum() * 1e-3) / 1e9
    fl = np.array(flush)
    rd = roofline("semkv_decode_attn (both pools in one kernel, FP16-block kernel, merge), one generation step",
                  float(np.mean(dbytes)), float(dec.mean()))
    quant_bytes = quant_algo_bytes(B, Lyr, H, prompt_tokens, nh_tok, nl_tok, wl.L_high, wl.L_low, T)
    rq = roofline("quantize_pack_kernel of the prompt (+ slot scan and counts)", quant_bytes, qms)
    res = _base_line(args, world, wl.name, world * dec_gbs,
                     tot_ms / G, {"B": B, "layers": Lyr, "kv_heads": H, "q_heads": H_q, "head_dim": 128,
                                  "prompt_len": "U[4096,16384] (seeded)", "prompt_tokens": prompt_tokens,
                                  "gen_steps": G, "block": 128, "L_high": wl.L_high, "L_low": wl.L_low,
                                  "r": wl.r_ppm / 1e6, "prompt_score": "attn_mass(w=64)",
                                  "token_score": "key_l2 of the new token at layer 31",
                                  "l2": "pools about 4 GB > 126 MB L2, no flush"},
                     clk, G * (1 + 1 + DECODE_LAUNCHES) + int(fl.sum()) * (1 + QUANT_LAUNCHES))
    res["steps"] = G
    res["value_is"] = "decode GB/s (pool rows + FP16 block read) over the 512 generation steps"
    res["components"] = {
        "tokens_per_s": round(world * B * G / (tot_ms * 1e-3), 1),
        "step_ms_mean": round(tot_ms / G, 4),
        "decode_ms_mean": round(float(dec.mean()), 4),
        "decode_gbs": round(dec_gbs, 1),
        "append_ms_median_no_flush": round(float(np.median(app[~fl])), 4),
        "block_flush_ms_median": round(float(np.median(app[fl])), 4) if fl.any() else None,
        "block_flushes": int(fl.sum()),
        "prompt_quantize_ms": round(qms, 4),
        "prompt_quantize_gbs_fp16_in": round(2 * Lyr * H * prompt_tokens * 256 / (qms * 1e-3) / 1e9, 1),
        "pool_capacity_note": "uniform per-sequence capacity sized for the longest prompt",
    }
    res["roofline"] = rd
    res["rooflines"] = {"decode": rd, "quantize_prompt": rq}
    return res


def run_long(args, rank, world, dist):
    """T = 131072, key-L2 score at layer 31; for each r: select, quantize
    (timed), 64 decode steps (timed)."""
    import torch

    import kv_cache_mixed_b200 as kv
    from inputs import synth
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    dev = torch.device("cuda")
    wl = synth.MISTRAL_LONG
    B, Lyr, H, H_q, T = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T
    stream = torch.cuda.current_stream()
    k, v = synth.kv(wl, 0, dev)
    seq_len = synth.seq_lens(wl, 0).to(dev)
    score = torch.empty((B, T), device=dev)
    mask = torch.empty((B, T), dtype=torch.uint8, device=dev)
    kv.semkv_score(kv.SCORE_KEY_L2, k[:, Lyr - 1], k.stride(0), None, seq_len, B, T, H, H_q, 64, score)
    nh_max = kv.semkv_num_high(T, max(synth.R_SWEEP_PPM))
    nl_max = T - kv.semkv_num_high(T, min(synth.R_SWEEP_PPM))
    cache = kv.MixedCache(B, Lyr, H, H_q, wl.L_high, wl.L_low, wl.r_ppm, nh_max + 16, nl_max + 16)
    qs = [synth.decode_query(wl, 0, dev, step=s) for s in range(64)]
    out = torch.empty_like(qs[0])
    fp16_in = 2 * B * Lyr * H * T * 256
    per_r = {}
    with Clocks(torch.cuda.current_device()) as clk:
        for r in synth.R_SWEEP_PPM:
            kv.semkv_select(score, seq_len, r, mask)

            def quant():
                cache.n_high.zero_()
                cache.n_low.zero_()
                kv.semkv_quantize(cache, k, v, seq_len, mask)
            qt = event_times(quant, args.warmup, args.steps, stream)
            it = iter(range(10 ** 9))
            dt = event_times(lambda: kv.semkv_decode_attn(cache, 0, Lyr, qs[next(it) % 64], out),
                             args.warmup, 64, stream)
            nh, nl = int(cache.n_high.sum().item()), int(cache.n_low.sum().item())
            qb = quant_algo_bytes(B, Lyr, H, B * T, nh, nl, wl.L_high, wl.L_low, T)
            db = decode_algo_bytes(Lyr, H, H_q, B, nh, nl, wl.L_high, wl.L_low, 0)
            qm, dm = statistics.median(qt), statistics.median(dt)
            rq, rd = roofline("quantize", qb, qm), roofline("decode", db, dm)
            per_r[str(r / 1e6)] = {"quantize_ms": round(qm, 4), "quantize_gbs_fp16_in": round(fp16_in / (qm * 1e-3) / 1e9, 1),
                                   "quantize_gbs_algorithmic": rq["achieved"], "quantize_frac": rq["frac"],
                                   "quantize_frac_vs_8TBs": rq["frac_vs_8TBs"],
                                   "decode_ms": round(dm, 4), "decode_gbs": rd["achieved"], "decode_frac": rd["frac"],
                                   "decode_frac_vs_8TBs": rd["frac_vs_8TBs"], "n_high": nh, "n_low": nl}
            if r == 500_000:
                head_q, head_rq, head_rd = qm, rq, rd
    assert cache.status_flags() == 0, "device status flags set"
    head_q = max_over_ranks(head_q, dist, dev)
    res = _base_line(args, world, wl.name, job_value(world, fp16_in, head_q), head_q,
                     {"B": B, "layers": Lyr, "kv_heads": H, "q_heads": H_q, "head_dim": 128, "T": T,
                      "L_high": wl.L_high, "L_low": wl.L_low, "r_sweep": [r / 1e6 for r in synth.R_SWEEP_PPM],
                      "score": "key_l2 at layer 31", "decode_steps": 64,
                      "l2": "inputs 16 GiB, pools > 3 GB: > 126 MB L2, no flush"},
                     clk, len(synth.R_SWEEP_PPM) * ((args.steps) * QUANT_LAUNCHES + 64 * DECODE_LAUNCHES))
    res["value_is"] = "quantize GB/s (FP16 in) at r = 0.5; per-r figures in components.per_r"
    res["components"] = {"per_r": per_r}
    res["roofline"] = head_rq
    res["rooflines"] = {"quantize": head_rq, "decode": head_rd}
    return res


def run_levels(args, rank, world, dist):
    """Batch 8, T = 32768, one layer, attention-mass score: quantize and decode
    per uniform level count and per adjacent pair (r = 0.5)."""
    import torch

    import kv_cache_mixed_b200 as kv
    from inputs import synth
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
    dev = torch.device("cuda")
    wl = synth.LEVEL_SWEEP
    B, Lyr, H, H_q, T, w = wl.B, wl.Lyr, wl.H, wl.H_q, wl.T, wl.w
    stream = torch.cuda.current_stream()
    k, v = synth.kv(wl, 0, dev)
    q_win = synth.q_window(wl, 0, dev)
    seq_len = synth.seq_lens(wl, 0).to(dev)
    score = torch.empty((B, T), device=dev)
    mask = torch.empty((B, T), dtype=torch.uint8, device=dev)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, 0], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    q = synth.decode_query(wl, 0, dev)
    out = torch.empty_like(q)
    fp16_in = 2 * B * Lyr * H * T * 256
    nh = kv.semkv_num_high(T, wl.r_ppm)
    per = {}
    with Clocks(torch.cuda.current_device()) as clk:
        for Lh, Ll in synth.LEVEL_PAIRS:
            cache = kv.MixedCache(B, Lyr, H, H_q, Lh, Ll, wl.r_ppm, nh + 16, T - nh + 16)

            def quant():
                cache.n_high.zero_()
                cache.n_low.zero_()
                kv.semkv_quantize(cache, k, v, seq_len, mask)
            qt = event_times(quant, args.warmup, args.steps, stream)
            dt = event_times(lambda: kv.semkv_decode_attn(cache, 0, Lyr, q, out), args.warmup, args.steps, stream)
            assert cache.status_flags() == 0, "device status flags set"
            nht, nlt = int(cache.n_high.sum().item()), int(cache.n_low.sum().item())
            qm, dm = statistics.median(qt), statistics.median(dt)
            rq = roofline("quantize", quant_algo_bytes(B, Lyr, H, B * T, nht, nlt, Lh, Ll, T), qm)
            rd = roofline("decode", decode_algo_bytes(Lyr, H, H_q, B, nht, nlt, Lh, Ll, 0), dm)
            key = f"{Lh}" if Lh == Ll else f"{Lh}/{Ll}"
            per[key] = {"quantize_ms": round(qm, 4), "quantize_gbs_fp16_in": round(fp16_in / (qm * 1e-3) / 1e9, 1),
                        "quantize_gbs_algorithmic": rq["achieved"], "quantize_frac": rq["frac"],
                        "quantize_frac_vs_8TBs": rq["frac_vs_8TBs"], "decode_ms": round(dm, 4),
                        "decode_gbs": rd["achieved"], "decode_frac": rd["frac"],
                        "decode_frac_vs_8TBs": rd["frac_vs_8TBs"],
                        "bytes_per_row_pair": pool_row_bytes(Lh) + pool_row_bytes(Ll)}
            if (Lh, Ll) == (6, 5):
                head_q, head_rq, head_rd = qm, rq, rd
            del cache
    head_q = max_over_ranks(head_q, dist, dev)
    res = _base_line(args, world, wl.name, job_value(world, fp16_in, head_q), head_q,
                     {"B": B, "layers": Lyr, "kv_heads": H, "q_heads": H_q, "head_dim": 128, "T": T,
                      "r": wl.r_ppm / 1e6, "levels": [f"{a}" if a == b else f"{a}/{b}" for a, b in synth.LEVEL_PAIRS],
                      "score": "attn_mass(w=64)", "l2": "inputs 1 GiB > 126 MB L2, no flush"},
                     clk, len(synth.LEVEL_PAIRS) * (args.warmup + args.steps) * (QUANT_LAUNCHES + DECODE_LAUNCHES))
    res["value_is"] = "quantize GB/s (FP16 in) at 6/5; per-level figures in components.per_level"
    res["components"] = {"per_level": per}
    res["roofline"] = head_rq
    res["rooflines"] = {"quantize": head_rq, "decode": head_rd}
    return res


# ------------------------------------------------------------------ CPU oracle
def oracle_step_sample(n_layers_sample=2):
    """Time the oracle on the default workload: the full score and select, and
    quantize+pack and decode for n_layers_sample of the 32 layers.  Returns
    (seconds, FP16 K+V bytes the sample quantized, description, cores used)."""
    import numpy as np

    from inputs import synth
    from oracle import semkv_oracle as O
    wl = synth.LLAMA_PREFILL
    layers = list(range(wl.Lyr - n_layers_sample, wl.Lyr))
    k, v = synth.kv(wl, 0, "cpu", layers=layers)
    q_win = synth.q_window(wl, 0, "cpu")
    qdec = synth.decode_query(wl, 0, "cpu")
    k, v, q_win, qdec = (t.numpy() for t in (k, v, q_win, qdec))
    T = wl.T

    def work():
        s = O.score_attn_mass(k[0, -1], q_win[0], T).astype(np.float32)
        mask = O.select_mask(s, O.num_high(T, wl.r_ppm))
        cache = O.MixedCache(1, n_layers_sample, wl.H, wl.L_high, wl.L_low, wl.r_ppm)
        cache.prefill(k, v, [T], [mask])
        cache.decode(qdec[:, layers])
    _, wall, cores, _ = cpu_cores_used(work)
    sample_bytes = 2 * n_layers_sample * wl.H * T * 256
    desc = (f"attention-mass score + select over all T={T}, then quantize+pack and decode of {n_layers_sample} "
            f"of {wl.Lyr} layers (all heads, all tokens); GB/s = FP16 K+V bytes of those {n_layers_sample} "
            f"layers / measured seconds ({wall:.1f} s)")
    return wall, sample_bytes, desc, cores


def cpu_baseline_json():
    # 7 of 32 layers: about 10-20 s of host work on the GPU machine
    wall, nbytes, desc, cores = oracle_step_sample(7)
    return {"value": round(nbytes / wall / 1e9, 4), "unit": "GB/s", "cores": cores,
            "threads_available": os.cpu_count(), "kind": "oracle", "sample": desc}


def cpu_baseline_workload(name):
    """The oracle on a bounded sample of a non-default workload."""
    import numpy as np

    from inputs import synth
    from oracle import semkv_oracle as O
    if name == "llama8b_generation_B16":
        wl = synth.GENERATION
        T = int(synth.seq_lens(wl, 0)[0])
        k, v = synth.kv(synth.scaled(wl, B=1), 0, "cpu", layers=[wl.Lyr - 1])
        q = synth.decode_query(synth.scaled(wl, B=1), 0, "cpu", n_layers=1).numpy()
        k, v = k.numpy()[:, :, :, :T], v.numpy()[:, :, :, :T]
        mask = (np.arange(T) % 2).astype(np.uint8)

        def work():
            c = O.MixedCache(1, 1, wl.H, wl.L_high, wl.L_low, wl.r_ppm)
            c.prefill(k, v, [T], [mask])
            t0 = time.perf_counter()
            c.decode(q)
            return time.perf_counter() - t0
        dsec, wall, cores, _ = cpu_cores_used(work)
        nbytes = 2 * wl.H * (T // 2 * pool_row_bytes(wl.L_high) + (T - T // 2) * pool_row_bytes(wl.L_low))
        return {"value": round(nbytes / dsec / 1e9, 4), "unit": "GB/s (decode, cache read)", "cores": cores,
                "threads_available": os.cpu_count(), "kind": "oracle",
                "sample": f"decode of sequence 0 (T={T}), layer 31, all 8 KV heads, from oracle pools "
                          f"({dsec:.1f} s of {wall:.1f} s)"}
    if name == "mistral7b_T131072":
        wl = synth.MISTRAL_LONG
        k, v = synth.kv(wl, 0, "cpu", layers=[wl.Lyr - 1])
        k, v = k.numpy(), v.numpy()
        T = wl.T
        mask = O.select_mask(O.score_key_l2(k[0, 0]), O.num_high(T, wl.r_ppm))

        def work():
            for x in (k, v):
                for h in range(wl.H):
                    O.quantize_slab(x[0, 0, h], mask, wl.L_high, wl.L_low)
        _, wall, cores, _ = cpu_cores_used(work)
        return {"value": round(2 * wl.H * T * 256 / wall / 1e9, 4), "unit": "GB/s (quantize, FP16 in)",
                "cores": cores, "threads_available": os.cpu_count(), "kind": "oracle",
                "sample": f"quantize+pack of layer 31 (K and V, 8 heads, T={T}) at r=0.5 ({wall:.1f} s)"}
    wl = synth.LEVEL_SWEEP
    k, v = synth.kv(synth.scaled(wl, B=1), 0, "cpu")
    k, v = k.numpy(), v.numpy()
    T = wl.T
    mask = (np.arange(T) % 2).astype(np.uint8)

    def work():
        for x in (k, v):
            for h in range(wl.H):
                O.quantize_slab(x[0, 0, h], mask, 6, 5)
    _, wall, cores, _ = cpu_cores_used(work)
    return {"value": round(2 * wl.H * T * 256 / wall / 1e9, 4), "unit": "GB/s (quantize, FP16 in)", "cores": cores,
            "threads_available": os.cpu_count(), "kind": "oracle",
            "sample": f"quantize+pack of sequence 0 (K and V, 8 heads, T={T}) at 6/5 ({wall:.1f} s)"}


def run_reference(args, rank):
    """The CPU oracle as the reference arm.  Each step is one bounded sample of
    the default workload (the full score and select, quantize+pack and decode
    of 1 of the 32 layers); value = FP16 K+V bytes of the sampled layer / the
    measured seconds, and ms_per_step is that measured time (nothing is
    extrapolated)."""
    if rank != 0:
        return None
    times, desc, cores, nbytes = [], "", 1.0, 0
    if args.warmup > 0:
        oracle_step_sample(1)
    for _ in range(max(1, args.steps)):
        wall, nbytes, desc, cores = oracle_step_sample(1)
        times.append(wall)
    per_step = statistics.median(times)
    value = nbytes / per_step / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": 1,
            "steps": max(1, args.steps), "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64 (numpy)",
            "data": "synthetic", "config": prefill_config(1),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "threads_available": os.cpu_count(), "kind": "oracle", "sample": desc},
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
    opts = {"quantize_rotated": {"rotate": True}, "quantize_pages": {"layout": kv.LAYOUT_PAGES}}.get(args.case, {})
    cache = kv.MixedCache(B, Lyr, H, H_q, wl.L_high, wl.L_low, wl.r_ppm, nh + 128, T - nh + 128, **opts)
    kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, Lyr - 1], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
    kv.semkv_select(score, seq_len, wl.r_ppm, mask)
    kv.semkv_quantize(cache, k, v, seq_len, mask)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    times = []
    for i in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if args.case == "score":
            kv.semkv_score(kv.SCORE_ATTN_MASS, k[:, Lyr - 1], k.stride(0), q_win, seq_len, B, T, H, H_q, w, score)
        elif args.case == "select":
            kv.semkv_select(score, seq_len, wl.r_ppm, mask)
        elif args.case.startswith("quantize"):
            cache.n_high.zero_()
            cache.n_low.zero_()
            kv.semkv_quantize(cache, k, v, seq_len, mask)
        else:
            kv.semkv_decode_attn(cache, 0, Lyr, qdec, out)
        b.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(a.elapsed_time(b))
    assert cache.status_flags() == 0
    print(json.dumps({"case": args.case, "layers": Lyr, "ok": True,
                      "ms_median": round(statistics.median(times), 4) if times else None}))


def main():
    args = parse()
    if args.case:
        run_case(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, dist = init_ranks("nccl")
    if args.workload == DEFAULT_WORKLOAD:
        res, state = run_prefill(args, rank, world, dist)
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
    else:
        fn = {"llama8b_generation_B16": run_generation, "mistral7b_T131072": run_long,
              "level_sweep_B8_T32768": run_levels}[args.workload]
        res = fn(args, rank, world, dist)
        res["e2e"] = None
        res["e2e_note"] = "end-to-end (host buffers) is measured on the default workload's line"
        if rank == 0 and world == 1 and not args.no_cpu:
            res["cpu_baseline"] = cpu_baseline_workload(args.workload)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
