#!/usr/bin/env python
"""Benchmark of the libropeattn hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  * prefill  rope_attn_fwd on the Llama-style GQA workload (B4 Hq32 Hkv8 S4096 D128, RoPE
    base 5e5, causal): RoPE table, K rotation, fused attention kernel;
  * decode   rope_attn_decode on the GQA decode workload (B32 Hq64 Hkv8, cache Sk 8192
    pre-rotated, query at position 8191): split-KV kernel and log-sum-exp combine.
The headline value is prefill TFLOP/s (causal FLOPs counted as 2*B*Hq*S^2*D); the decode
leg is reported beside it in GB/s of algorithmic HBM bytes (K and V cache read once, q
read, out written). Inputs are resident in HBM when the timed region starts; every step
streams the 1.07 GB KV cache, far larger than the 126 MB L2, so no step finds the previous
step's prefill inputs in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 (one process per GPU under torch.distributed.run): every rank runs its own batch of
the same shapes (weak scaling, no data-path collective); the barrier and the max over ranks
bracket the timed region. --impl reference times the fp64 CPU oracle (the baseline arm).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from synthetic import DECODE, LLAMA, LONG, Workload, make_inputs  # noqa: E402

PREFILL_W, DECODE_W = LLAMA, DECODE
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_BF16_TFLOPS, SPEC_HBM_GBS = 2250.0, 8000.0
KERNEL_SOURCES = {
    "attn_fwd_sm100_kernel": ["transformer_attention_04_b200/csrc/attn_fwd_sm100.cuh",
                              "transformer_attention_04_b200/csrc/ptx.cuh"],
    "decode_split_kernel": ["transformer_attention_04_b200/csrc/decode.cuh",
                            "transformer_attention_04_b200/csrc/ptx.cuh"],
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--prewarm-s", type=float, default=0.5,
                    help="seconds of untimed steps before the counted warm-up (0 for profiler runs)")
    ap.add_argument("--skip-next", action="store_true",
                    help="skip the sliding-window / KV-cache / paged decode measurements")
    ap.add_argument("--profile-leg", choices=["prefill", "decode", "window", "paged", "ring"],
                    default=None,
                    help="run only this leg, warm-up + steps launches, and print no JSON "
                         "(the command that ncu captures wraps; holds only that leg's buffers)")
    a = ap.parse_args(argv)
    a.warmup = max(a.warmup, 3)
    return a


# ----------------------------------------------------------------------------- ranks

def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local, backend="nccl"):
    if world > 1:
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(values, world, device=None):
    """Element-wise max of a list of floats over all ranks (identity when world == 1)."""
    if world == 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_seed(rank: int, leg: int) -> int:
    """Each rank draws its own batch: the same shapes, a distinct seed per rank and leg."""
    return 1000 * leg + rank


# ----------------------------------------------------------------------------- helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str):
    """sha256[:16] over the code of the source files a kernel is compiled from (comments
    removed and whitespace collapsed, so only a change to the code itself counts)."""
    import re
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, p)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel]
        if e.get("source_hash") != kernel_source_hash(kernel.split()[0]):
            return None
        return int(e["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_prefill_sample(rows_from_end: int):
    """The fp64 oracle (as it stands) on query rows of batch 0, head 0 of the prefill
    workload: the last ``rows_from_end`` rows (each row of attention is independent, so a
    row subset is an exact piece of the job; its FLOPs are counted per row)."""
    from synthetic import Workload, to_f64
    w1 = Workload("prefill sample", 1, 1, 1, PREFILL_W.Sq, PREFILL_W.Sk, PREFILL_W.D,
                  PREFILL_W.rope_base)
    q, k, v = (to_f64(t) for t in make_inputs(w1, 0))
    S, D = PREFILL_W.Sq, PREFILL_W.D
    rows = np.arange(S - rows_from_end, S)
    flops = 4 * D * int(np.sum(rows + 1))  # row i attends i + 1 keys: QK^T and PV
    return (q, k, v, rows), flops


def run_oracle_prefill(sample):
    import oracle
    q, k, v, rows = sample
    t0 = time.perf_counter()
    oracle.rope_attn_fwd(q, k, v, PREFILL_W.rope_base, 0, True, rows=rows)
    return time.perf_counter() - t0


def oracle_decode_time():
    """The oracle on batch element 0 of the decode workload (64 heads, 8192 keys)."""
    import oracle
    from synthetic import Workload, to_f64
    wd = Workload("decode sample", 1, DECODE_W.Hq, DECODE_W.Hkv, 1, DECODE_W.Sk, DECODE_W.D,
                  DECODE_W.rope_base, decode_pos=DECODE_W.decode_pos)
    qd, kd, vd = (to_f64(t) for t in make_inputs(wd, 1))
    t0 = time.perf_counter()
    oracle.rope_attn_decode(qd, kd, vd, wd.rope_base, wd.decode_pos)
    return wd, time.perf_counter() - t0


def pick_rows(budget_s: float) -> int:
    """Largest multiple of 128 rows (counted from the end of one head) whose oracle time
    fits in ``budget_s``, from one calibration run of 128 rows."""
    sample, _ = oracle_prefill_sample(128)
    t128 = run_oracle_prefill(sample)
    rows = int(max(1, budget_s / max(t128, 1e-3))) * 128
    return max(128, min(PREFILL_W.Sq, rows))


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    world, rank, _ = dist_info()
    if rank != 0:
        return 0
    # every step is a bounded sample sized so the whole run stays near two minutes
    budget = min(15.0, 120.0 / (args.warmup + args.steps))
    rows = pick_rows(budget)
    sample, flops = oracle_prefill_sample(rows)
    tp = [run_oracle_prefill(sample) for _ in range(args.warmup + args.steps)][args.warmup:]
    wd, td = oracle_decode_time()
    value = flops * len(tp) / sum(tp) / 1e12
    cores = blas_threads()
    desc = (f"prefill: last {rows} query rows of batch 0 head 0 of {PREFILL_W.name} "
            f"(of {PREFILL_W.B * PREFILL_W.Hq} heads x {PREFILL_W.Sq} rows), per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sum(tp) / len(tp), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(world),
        "decode": {"value": wd.io_bytes() / td / 1e9, "unit": "GB/s",
                   "sample": "batch 0 of the decode workload, once"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


METRIC = "RoPE causal GQA attn TFLOP/s & % BF16 peak; decode KV-read GB/s & % HBM"


def config_block(world):
    return {
        "workload": (f"{PREFILL_W.name} B{PREFILL_W.B} Hq{PREFILL_W.Hq} Hkv{PREFILL_W.Hkv} "
                     f"S{PREFILL_W.Sq} D{PREFILL_W.D} base {PREFILL_W.rope_base:g} causal + "
                     f"{DECODE_W.name} B{DECODE_W.B} Hq{DECODE_W.Hq} Hkv{DECODE_W.Hkv} "
                     f"Sk{DECODE_W.Sk} D{DECODE_W.D} pos {DECODE_W.decode_pos}"),
        "prefill": {"B": PREFILL_W.B, "Hq": PREFILL_W.Hq, "Hkv": PREFILL_W.Hkv, "S": PREFILL_W.Sq,
                    "D": PREFILL_W.D, "rope_base": PREFILL_W.rope_base, "causal": True},
        "decode": {"B": DECODE_W.B, "Hq": DECODE_W.Hq, "Hkv": DECODE_W.Hkv, "Sk": DECODE_W.Sk,
                   "D": DECODE_W.D, "pos": DECODE_W.decode_pos},
        "inputs": "iid N(0,1) rounded to bf16, seeded per rank",
        "l2": "not flushed: each step streams the 1.07 GB KV cache (> 126 MB L2)",
        "parallelism": "single GPU" if world == 1 else f"{world} independent replicas (weak)",
    }


def run_ours(args):
    import transformer_attention_04_b200 as ra
    world, rank, local = dist_info()
    init_dist(world, local)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    qp, kp, vp = make_inputs(PREFILL_W, rank_seed(rank, 0))
    qd, kd, vd = make_inputs(DECODE_W, rank_seed(rank, 1))
    g_qp, g_kp, g_vp = (t.to(dev) for t in (qp, kp, vp))
    g_qd, g_kd, g_vd = (t.to(dev) for t in (qd, kd, vd))
    op = torch.empty_like(g_qp)
    od = torch.empty_like(g_qd)
    W = PREFILL_W
    # K rotation, attention | decode split, combine (the cos/sin table is built at the first
    # call and kept, so no table launch falls inside the timed region)
    launches_per_step = 4

    def step(evs=None):
        if evs:
            evs[0].record()
        ra.rope_attn_fwd(g_qp, g_kp, g_vp, W.rope_base, 0, True, out=op)
        if evs:
            evs[1].record()
        ra.rope_attn_decode(g_qd, g_kd, g_vd, DECODE_W.rope_base, DECODE_W.decode_pos, out=od)
        if evs:
            evs[2].record()

    vis = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    sampler = ClockSampler(vis[local] if local < len(vis) else local).start()
    # a freshly leased GPU runs its first ~50 ms of work slow (clock and power ramp): steps
    # are run untimed for at least --prewarm-s seconds before the counted warm-up steps
    if args.prewarm_s > 0:
        prewarm(step, args.prewarm_s)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ra.rope_attn_get_device_status() != ra.RA_OK:
        raise RuntimeError("device timeout during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # torch creates an event at its first record: record every one once now, so that the
    # timed loop only re-records them (the library's profiling pairs are made at enable)
    for e in [t_start, t_end] + [x for trio in evs for x in trio]:
        e.record()
    ra.rope_attn_profile_enable(True)
    barrier(world)
    torch.cuda.synchronize()
    # the library's kernel events sit between a call's kernels, where they hold back the
    # programmatic overlap of each kernel's start with the previous one's end: odd steps carry
    # them (the kernel rooflines), even steps run as a user's calls do (the call figures)
    K = args.steps
    profiled = [K == 1 or i % 2 == 1 for i in range(K)]
    t_start.record()
    host_s = []
    for i in range(K):
        ra.rope_attn_profile_pause(not profiled[i])
        h0 = time.perf_counter()
        step(evs[i])
        host_s.append(time.perf_counter() - h0)
    t_end.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    k_ms, k_n = ra.rope_attn_profile_read(0)
    d_ms, d_n = ra.rope_attn_profile_read(1)
    ra.rope_attn_profile_enable(False)
    if ra.rope_attn_get_device_status() != ra.RA_OK:
        raise RuntimeError("device timeout in the timed region")

    total_ms = t_start.elapsed_time(t_end)
    plain = [e for e, pr in zip(evs, profiled) if not pr]
    timing = (f"value and the call figures: the {len(plain)} timed steps without kernel events; "
              f"roofline: the library's kernel events of the other {K - len(plain)}"
              if plain else "one timed step: calls timed with the kernel events inside")
    plain = plain or evs
    n_calls = len(plain)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in plain)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in plain)
    total_ms, pre_ms, dec_ms, k_ms, d_ms = max_over_ranks([total_ms, pre_ms, dec_ms, k_ms, d_ms],
                                                          world, dev)
    peaks, peak_src = measured_peaks()
    value = world * W.flops() * n_calls / (pre_ms * 1e-3) / 1e12
    dec_gbs = world * DECODE_W.io_bytes() * n_calls / (dec_ms * 1e-3) / 1e9
    attn_tflops = W.flops() / (k_ms / k_n * 1e-3) / 1e12
    split_gbs = DECODE_W.io_bytes() / (d_ms / d_n * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_block(world),
        "frac_spec_bf16": value / world / SPEC_BF16_TFLOPS,
        "decode": {"value": dec_gbs, "unit": "GB/s", "us_per_call": 1e3 * dec_ms / n_calls,
                   "frac_spec_hbm": dec_gbs / world / SPEC_HBM_GBS,
                   "splits": ra.rope_attn_decode_auto_splits(DECODE_W.B, DECODE_W.Hq, DECODE_W.Hkv,
                                                             DECODE_W.Sk, DECODE_W.D,
                                                             DECODE_W.decode_pos),
                   "roofline": {"bound": "hbm", "achieved": split_gbs, "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": split_gbs / peaks["hbm_gbs"],
                                "peak_source": peak_src,
                                "kernel": "decode_split_kernel<128, false>",
                                "traffic": recorded_traffic("decode_split_kernel decode")}},
        "prefill_ms_per_call": pre_ms / n_calls,
        "call_timing": timing,
        # the host's own cost per step: the median over the first steps, which run before
        # the launch queue fills (later enqueues wait for the GPU to free queue space)
        "host_us_per_step": 1e6 * statistics.median(host_s[:20]),
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16_tflops"],
                     "peak_source": f"{peak_src} burst bf16 GEMM",
                     "frac_sustained": attn_tflops / peaks["bf16_tflops_sustained"],
                     "kernel": "attn_fwd_sm100_kernel<128>", "launches": k_n,
                     "ms_per_launch": k_ms / k_n,
                     "traffic": recorded_traffic("attn_fwd_sm100_kernel llama")},
        "clocks": clocks,
        "gpu_launches": launches_per_step * K,
    }

    if not args.skip_e2e:
        line["e2e"] = e2e_leg(ra, args, world, dev, qp, kp, vp, qd, kd, vd)
    if not args.skip_next:
        del g_qp, g_kp, g_vp, g_qd, g_kd, g_vd, op, od
        line["next_rows"] = next_rows_leg(ra, world, rank, dev, peaks)
    if world == 1 and rank == 0 and not args.skip_cpu_baseline:
        rows = pick_rows(6.0)
        sample, flops = oracle_prefill_sample(rows)
        tp = [run_oracle_prefill(sample) for _ in range(2)]
        wd, td = oracle_decode_time()
        line["cpu_baseline"] = {
            "value": flops * len(tp) / sum(tp) / 1e12, "unit": "TFLOP/s",
            "cores": blas_threads(), "kind": "oracle",
            "sample": (f"prefill: last {rows} query rows of batch 0 head 0 (of "
                       f"{PREFILL_W.B * PREFILL_W.Hq} heads x {PREFILL_W.Sq} rows), timed twice; "
                       f"decode: batch 0 of {DECODE_W.B} at {wd.io_bytes() / td / 1e9:.3f} GB/s"),
        }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def window_pairs(S: int, W: int) -> int:
    """(query, key) pairs a causal sliding window of W allows over S tokens: sum_i min(i+1, W)."""
    if W <= 0 or W >= S:
        return S * (S + 1) // 2
    return W * (W + 1) // 2 + (S - W) * W


def prewarm(fn, seconds: float) -> int:
    """Call fn() back to back until `seconds` of device time have passed; returns the calls."""
    n, t0 = 0, time.perf_counter()
    while True:
        for _ in range(8):
            fn()
        n += 8
        torch.cuda.synchronize()
        if time.perf_counter() - t0 >= seconds:
            return n


def time_calls(fn, reps: int, warm: int = 3) -> float:
    """Mean device milliseconds of fn() over reps back-to-back calls (CUDA events)."""
    prewarm(fn, 0.2)
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


WINDOW_W = 4096  # the sliding-window row: W = 4096 over the 32k-token workload
PAGE = 16  # the paged row: 16-token pages


RING_RANKS = 8  # the ring row: the 32k-token workload over 8 ranks (4096 tokens each)


def ring_local_timed(ra, Wl, q, k, v, reps: int, layout: str = "contiguous"):
    """Time the attention phase of an 8-rank ring run rank after rank on this GPU (every
    rank's partial-attention calls in its ring order; key rotation and slicing excluded).
    Returns (ms per pass, per-rank ms of the last pass)."""
    evs = {}

    def hook(r, phase):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        evs[(r, phase)] = e

    ra.ring_attention_local(q, k, v, Wl.rope_base, RING_RANKS, True, layout=layout)
    total, per = 0.0, []
    for _ in range(reps):
        evs.clear()
        ra.ring_attention_local(q, k, v, Wl.rope_base, RING_RANKS, True, on_rank=hook,
                                layout=layout)
        torch.cuda.synchronize()
        total += evs[(0, "start")].elapsed_time(evs[(RING_RANKS - 1, "end")])
        per = [evs[(r, "start")].elapsed_time(evs[(r, "end")]) for r in range(RING_RANKS)]
    return total / reps, per


def decode_step_inputs(Dw, rank, dev):
    """The decode-step rows' inputs: the decode workload's q and cache, a new token per
    sequence, positions 8191 - 128 b (4223..8191) and the cache split into 16-token pages of a
    shuffled pool (block table a seeded permutation)."""
    q, kc, vc = (t.to(dev) for t in make_inputs(Dw, rank_seed(rank, 1)))
    g = torch.Generator().manual_seed(rank_seed(rank, 3))
    kn = torch.randn(Dw.B, Dw.Hkv, 1, Dw.D, generator=g).to(torch.bfloat16).to(dev)
    vn = torch.randn(Dw.B, Dw.Hkv, 1, Dw.D, generator=g).to(torch.bfloat16).to(dev)
    pos_h = [Dw.Sk - 1 - 128 * b for b in range(Dw.B)]
    pos = torch.tensor(pos_h, dtype=torch.int32, device=dev)
    per = Dw.Sk // PAGE
    perm = torch.randperm(Dw.B * per, generator=g).to(torch.int32)
    table = perm.view(Dw.B, per).to(dev)
    return q, kc, vc, kn, vn, pos, pos_h, table


def to_pages(Dw, cache, table):
    """Scatter a contiguous [B, Hkv, Sk, D] cache into a pool [B*Sk/PAGE, Hkv, PAGE, D] by the
    block table."""
    per = Dw.Sk // PAGE
    pool = torch.empty(Dw.B * per, Dw.Hkv, PAGE, Dw.D, dtype=cache.dtype, device=cache.device)
    pool[table.view(-1).long()] = cache.view(Dw.B, Dw.Hkv, per, PAGE, Dw.D).permute(
        0, 2, 1, 3, 4).reshape(-1, Dw.Hkv, PAGE, Dw.D)
    return pool


def next_rows_leg(ra, world, rank, dev, peaks):
    """The rows after the headline path, each timed on its own with CUDA events:
    sliding-window prefill (W = 4096 over the 32k-token workload); the same workload causal in
    one call, and as a ring of 8 ranks run in turn (contiguous and zig-zag); chunked prefill
    into a KV cache (the Llama prefill written into a cache); odd group sizes; the decode step
    with in-kernel append at per-sequence positions, and the same step on a paged cache
    (16-token pages)."""
    res = {}
    # sliding window: FLOPs count only the allowed pairs (4*D per pair: Q.K and P.V)
    Wl, W = LONG, WINDOW_W
    q, k, v = (t.to(dev) for t in make_inputs(Wl, rank_seed(rank, 2)))
    out = torch.empty_like(q)
    ms = time_calls(lambda: ra.rope_attn_prefill(q, k, v, Wl.rope_base, 0, True, window=W,
                                                 out=out), 5)
    flops = 4 * Wl.D * Wl.B * Wl.Hq * window_pairs(Wl.Sq, W)
    res["sliding_window_prefill"] = _rate_entry(
        f"{Wl.name} B{Wl.B} Hq{Wl.Hq} Hkv{Wl.Hkv} S{Wl.Sq} D{Wl.D} causal, window {W}", ms, flops,
        world, "tensor", peaks["bf16_tflops"], 1e12, "TFLOP/s", "attn_fwd_sm100_kernel window")
    # the same workload as one causal call on one GPU (the long-context configuration itself)
    ms = time_calls(lambda: ra.rope_attn_fwd(q, k, v, Wl.rope_base, 0, True, out=out), 3)
    res["long_context_prefill"] = _rate_entry(
        f"{Wl.name} B{Wl.B} Hq{Wl.Hq} Hkv{Wl.Hkv} S{Wl.Sq} D{Wl.D} causal, one call", ms,
        Wl.flops(), world, "tensor", peaks["bf16_tflops"], 1e12, "TFLOP/s")
    # ring attention: the same workload, causal, as an 8-rank ring whose ranks run in turn
    # here; per-rank times give the compute of each rank in a real ring
    ms, per_rank = ring_local_timed(ra, Wl, q, k, v, 3)
    L = Wl.Sk // RING_RANKS
    e = _rate_entry(
        f"{Wl.name} B{Wl.B} Hq{Wl.Hq} Hkv{Wl.Hkv} S{Wl.Sq} D{Wl.D} causal as a {RING_RANKS}-rank "
        f"ring ({L} tokens per rank), ranks run in turn on one GPU", ms, Wl.flops(), world,
        "tensor", peaks["bf16_tflops"], 1e12, "TFLOP/s")
    e["per_rank_ms"] = per_rank
    e["critical_rank_ms"] = max(per_rank)
    e["exchange_bytes_per_step"] = 2 * Wl.B * Wl.Hkv * L * Wl.D * 2
    e["kernel"] = "attn_fwd_sm100_kernel"
    e["block_traffic"] = recorded_traffic("attn_fwd_sm100_kernel ring")
    res["ring_long_context_8_ranks"] = e
    # the same ring with the zig-zag split (rank r holds chunks r and 15 - r of 2048 tokens):
    # every rank attends the same number of chunk blocks
    ms, per_rank = ring_local_timed(ra, Wl, q, k, v, 3, layout="zigzag")
    e = _rate_entry(
        f"{Wl.name} B{Wl.B} Hq{Wl.Hq} Hkv{Wl.Hkv} S{Wl.Sq} D{Wl.D} causal as a {RING_RANKS}-rank "
        f"zig-zag ring (chunks of {L // 2} tokens, rank r holds chunks r and "
        f"{2 * RING_RANKS - 1}-r), ranks run in turn on one GPU", ms, Wl.flops(), world,
        "tensor", peaks["bf16_tflops"], 1e12, "TFLOP/s")
    e["per_rank_ms"] = per_rank
    e["critical_rank_ms"] = max(per_rank)
    e["exchange_bytes_per_step"] = 2 * Wl.B * Wl.Hkv * L * Wl.D * 2
    res["ring_long_context_8_ranks_zigzag"] = e
    del q, k, v, out
    # chunked prefill into a cache: the headline prefill with its keys/values written out
    P = PREFILL_W
    q, k, v = (t.to(dev) for t in make_inputs(P, rank_seed(rank, 0)))
    kc = torch.empty(P.B, P.Hkv, P.Sk + 512, P.D, dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    out = torch.empty_like(q)
    ms = time_calls(lambda: ra.rope_attn_prefill(q, k, v, P.rope_base, 0, True, k_cache_rot=kc,
                                                 v_cache=vc, out=out), 20)
    res["prefill_into_cache"] = _rate_entry(
        f"{P.name} B{P.B} Hq{P.Hq} Hkv{P.Hkv} S{P.Sq} D{P.D} causal into a {P.Sk + 512}-row cache",
        ms, P.flops(), world, "tensor", peaks["bf16_tflops"], 1e12, "TFLOP/s")
    del q, k, v, out, kc, vc
    # other head groupings at the Llama shape: an odd group size (G = 3, whose units pair
    # two consecutive query tiles of one head) and multi-query attention (8 query heads on
    # one key/value head)
    for key, (Bg, Hqg, Hkvg) in (("gqa_group3_prefill", (4, 24, 8)),
                                 ("mqa_group8_prefill", (4, 8, 1))):
        Wg = Workload(f"{P.name} G{Hqg // Hkvg}", Bg, Hqg, Hkvg, P.Sq, P.Sk, P.D, P.rope_base)
        q, k, v = (t.to(dev) for t in make_inputs(Wg, rank_seed(rank, 3)))
        out = torch.empty_like(q)
        ms = time_calls(lambda: ra.rope_attn_fwd(q, k, v, Wg.rope_base, 0, True, out=out), 20)
        res[key] = _rate_entry(
            f"causal prefill B{Bg} Hq{Hqg} Hkv{Hkvg} (G = {Hqg // Hkvg}) S{P.Sq} D{P.D}", ms,
            Wg.flops(), world, "tensor", peaks["bf16_tflops"], 1e12, "TFLOP/s")
        del q, k, v, out
    # decode step with append at per-sequence positions, contiguous and paged
    Dw = DECODE_W
    q, kc, vc, kn, vn, pos, pos_h, table = decode_step_inputs(Dw, rank, dev)
    rows = sum(p + 1 for p in pos_h)
    nbytes = (2 * rows * Dw.Hkv * Dw.D * 2 + 2 * Dw.B * Dw.Hq * Dw.D * 2 +
              4 * Dw.B * Dw.Hkv * Dw.D * 2)  # K,V rows read; q, out; new token read + written
    od = torch.empty_like(q)
    ms = time_calls(lambda: ra.rope_attn_decode_step(q, kc, vc, pos, max(pos_h), Dw.rope_base, kn,
                                                     vn, out=od), 50)
    work = (f"{Dw.name} B{Dw.B} Hq{Dw.Hq} Hkv{Dw.Hkv} D{Dw.D}, positions 8191 - 128 b "
            f"(4223..8191), new token appended")
    res["decode_step_varlen_append"] = _rate_entry(work, ms, nbytes, world, "hbm",
                                                   peaks["hbm_gbs"], 1e9, "GB/s")
    kp, vp = to_pages(Dw, kc, table), to_pages(Dw, vc, table)
    del kc, vc
    ms = time_calls(lambda: ra.rope_attn_decode_paged(q, kp, vp, table, pos, max(pos_h),
                                                      Dw.rope_base, kn, vn, out=od), 50)
    res["paged_decode_append"] = _rate_entry(work + f", {PAGE}-token pages in a shuffled pool", ms,
                                             nbytes, world, "hbm", peaks["hbm_gbs"], 1e9, "GB/s",
                                             "decode_split_kernel paged")
    del q, kp, vp, od
    torch.cuda.synchronize()
    if ra.rope_attn_get_device_status() != ra.RA_OK:
        raise RuntimeError("device status error in the next-rows leg")
    # every rank reports the slowest rank's time
    keys = list(res)
    worst = max_over_ranks([res[k]["ms_per_call"] for k in keys], world, dev)
    for k, t in zip(keys, worst):
        e = res[k]
        e["ms_per_call"] = t
        e["value"] = world * e["work_per_call"] / (t * 1e-3) / e.pop("_scale")
        e["frac_of_measured_peak"] = e["value"] / world / e["peak"]
    return res


def _rate_entry(workload, ms, work, world, bound, peak, scale, unit, traffic_key=None):
    e = {"workload": workload, "ms_per_call": ms, "work_per_call": work, "unit": unit,
         "bound": bound, "peak": peak, "_scale": scale,
         "note": "inputs resident in HBM; mean over back-to-back calls (CUDA events)"}
    if traffic_key:
        # DRAM bytes of the call's main kernel from its committed ncu capture (null once the
        # kernel's code has changed since)
        e["kernel"] = traffic_key.split()[0]
        e["traffic"] = recorded_traffic(traffic_key)
    return e


def e2e_leg(ra, args, world, dev, qp, kp, vp, qd, kd, vd):
    """The same metric through the public API from pinned HOST buffers: every step copies
    its inputs host->device, runs the call and copies the result back."""
    pins = [t.pin_memory() for t in (qp, kp, vp, qd, kd, vd)]
    outs_h = [torch.empty_like(qp).pin_memory(), torch.empty_like(qd).pin_memory()]
    W = PREFILL_W
    h2d = sum(t.numel() * t.element_size() for t in pins)
    d2h = sum(t.numel() * t.element_size() for t in outs_h)
    times_p, times_d = [], []
    for it in range(1 + args.e2e_steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        torch.cuda.synchronize()
        e[0].record()
        gq, gk, gv = (t.to(dev, non_blocking=True) for t in pins[:3])
        o = ra.rope_attn_fwd(gq, gk, gv, W.rope_base, 0, True)
        outs_h[0].copy_(o, non_blocking=True)
        e[1].record()
        gqd, gkd, gvd = (t.to(dev, non_blocking=True) for t in pins[3:])
        od = ra.rope_attn_decode(gqd, gkd, gvd, DECODE_W.rope_base, DECODE_W.decode_pos)
        outs_h[1].copy_(od, non_blocking=True)
        e[2].record()
        torch.cuda.synchronize()
        del gq, gk, gv, gqd, gkd, gvd, o, od
        if it > 0:
            times_p.append(e[0].elapsed_time(e[1]))
            times_d.append(e[1].elapsed_time(e[2]))
    tp, td = max_over_ranks([sum(times_p), sum(times_d)], world, dev)
    n = len(times_p)
    return {"value": world * W.flops() * n / (tp * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": (tp + td) / n,
            "decode_gbs": world * DECODE_W.io_bytes() * n / (td * 1e-3) / 1e9,
            "steps": n}


def run_profile_leg(args):
    """One leg alone, for profiler captures: the same inputs and calls as the timed step."""
    import transformer_attention_04_b200 as ra
    dev = torch.device("cuda", 0)
    if args.profile_leg == "prefill":
        W = PREFILL_W
        q, k, v = (t.to(dev) for t in make_inputs(W, rank_seed(0, 0)))
        out = torch.empty_like(q)
        call = lambda: ra.rope_attn_fwd(q, k, v, W.rope_base, 0, True, out=out)
    elif args.profile_leg == "decode":
        W = DECODE_W
        q, k, v = (t.to(dev) for t in make_inputs(W, rank_seed(0, 1)))
        out = torch.empty_like(q)
        call = lambda: ra.rope_attn_decode(q, k, v, W.rope_base, W.decode_pos, out=out)
    elif args.profile_leg == "window":
        W = LONG
        q, k, v = (t.to(dev) for t in make_inputs(W, rank_seed(0, 2)))
        out = torch.empty_like(q)
        call = lambda: ra.rope_attn_prefill(q, k, v, W.rope_base, 0, True, window=WINDOW_W,
                                            out=out)
    elif args.profile_leg == "ring":
        # one pass = the 36 partial-attention launches of the 8-rank ring (plus 8 rotations)
        W = LONG
        q, k, v = (t.to(dev) for t in make_inputs(W, rank_seed(0, 2)))
        call = lambda: ra.ring_attention_local(q, k, v, W.rope_base, RING_RANKS, True)
    else:
        W = DECODE_W
        q, kc, vc, kn, vn, pos, pos_h, table = decode_step_inputs(W, 0, dev)
        kp, vp = to_pages(W, kc, table), to_pages(W, vc, table)
        del kc, vc
        out = torch.empty_like(q)
        call = lambda: ra.rope_attn_decode_paged(q, kp, vp, table, pos, max(pos_h), W.rope_base,
                                                 kn, vn, out=out)
    for _ in range(args.warmup + args.steps):
        call()
    torch.cuda.synchronize()
    st = ra.rope_attn_get_device_status()
    print(f"{args.profile_leg}: {args.warmup + args.steps} calls, device status {st}", flush=True)
    return 0 if st == ra.RA_OK else 1


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_leg:
        return run_profile_leg(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
