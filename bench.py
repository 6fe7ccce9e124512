"""Benchmark: exact attention forward TFLOP/s on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one forward over the whole workload (default: causal B4 H32 N8192
D128 bf16).  `value` is the whole-job TFLOP/s (4*B*H*N_q*N_k*D times the
fraction of 128x128 blocks with a visible pair, per step, summed over ranks,
divided by the slowest rank's CUDA-event time for K steps).  Inputs are
resident in HBM and larger than L2.  `e2e` measures the same metric through
fa_fwd_host with pinned host buffers, host<->device copies inside the timed
region.  With N > 1 each rank runs its own batch of the workload (weak
scaling; the work units are independent, so there is no collective on the
data path).

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).

--backward times the backward instead (fa_bwd: dQ, dK, dV from a fixed
forward's O and LSE and a random dO), credited 2.5x the forward's FLOP (five
matrix products per block against two).
"""

from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_attention_136_b200 import workloads as W  # noqa: E402
from exact_attention_136_b200 import inputs  # noqa: E402

METRIC = "attention fwd TFLOP/s and % of dense tensor peak (1×B200) vs CPU oracle"
METRIC_BWD = "attention bwd TFLOP/s and % of dense tensor peak (1×B200) vs CPU oracle"
BWD_FLOP_RATIO = 2.5
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_TFLOPS = {"fp16": 2250.0, "bf16": 2250.0, "e4m3": 4500.0}
PROFILE_DIR = os.path.join(ROOT, "profiles")
# the forward kernel and its host code (the backward's sources are not part of it)
KERNEL_SOURCES = ["exact_attention_136_b200/csrc/fa_fwd_kernel.cuh", "exact_attention_136_b200/csrc/sm100.cuh",
                  "exact_attention_136_b200/csrc/fa_api.cu", "exact_attention_136_b200/csrc/tmap.h"]


def kernel_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seeds(w: W.Workload, rank: int):
    """Seeds of this rank's batch: every rank draws its own inputs (weak scaling)."""
    return tuple(s + 7919 * rank for s in w.seeds)


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank float over the process group (the value itself with one process)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks(dtype: str):
    """(peak TF/s for the kernel timed alone, source string, sustained) from MEASURED_PEAKS.json."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    ratio = 2.0 if dtype == "e4m3" else 1.0
    try:
        with open(path) as f:
            mp = json.load(f)
        return mp["bf16_tflops"] * ratio, "measured", mp.get("bf16_tflops_sustained", None)
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS * ratio, "fallback", None


def recorded_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel."""
    path = os.path.join(PROFILE_DIR, "fa_fwd_kernel_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(workload)
    if not entry or entry.get("kernel_hash") != kernel_hash():
        return None
    return entry.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            text, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            text, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(text)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def graph_ms(fn, dev, n=20, reps=10):
    """Milliseconds per call of fn(stream) with the host out of the way: n calls captured in one
    CUDA graph on a side stream (after three warm-up calls there), replayed `reps` times between
    CUDA events on that stream."""
    cs = torch.cuda.Stream(dev)
    cs.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(cs):
        for _ in range(3):
            fn(cs)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        for _ in range(n):
            fn(cs)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(cs):
        g.replay()
        e0.record(cs)
        for _ in range(reps):
            g.replay()
        e1.record(cs)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / (n * reps)
    del g
    return ms


def standard_attention_context(w: W.Workload, q, k, v, ms_ours: float, dev, stream):
    """Informative only, for non-causal unmasked 16-bit workloads: the pages' "standard attention"
    ((q @ k^T * scale).softmax(-1) @ v in the input type, torch eager on cuBLAS; Flash Attention |
    Hermes Skill, Workflow 1, Step 3) and torch's scaled_dot_product_attention (the pages' flash
    call, a library kernel) on the same inputs and GPU, each timed with CUDA events after warm-up.
    Neither is a target or an oracle; `speedup` = their time / this library's."""
    if w.causal or w.window_left >= 0 or w.mask or w.dtype not in ("fp16", "bf16") or w.h_kv != w.H:
        return None
    qt, kt, vt = (t.transpose(1, 2) for t in (q, k, v))   # [B, H, N, D] views, as the pages' snippet

    def standard():
        return (qt @ kt.transpose(-2, -1) * w.scale).softmax(dim=-1) @ vt

    def sdpa():
        return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=w.scale)

    res = {}
    with torch.cuda.stream(stream):
        for name, fn in (("standard_attention", standard), ("sdpa", sdpa)):
            try:
                for _ in range(3):
                    fn()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(20):
                    fn()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                ms = e0.elapsed_time(e1) / 20
                res[name] = {"ms": ms, "speedup": ms / ms_ours}
            except (RuntimeError, torch.cuda.OutOfMemoryError) as exc:
                res[name] = {"unavailable": str(exc).splitlines()[0][:200]}
    # the same three with the host out of the way (CUDA-graph replays): launch-bound shapes
    from exact_attention_136_b200 import forward
    try:
        ours_g = graph_ms(lambda s: forward(q, k, v, w.scale, False, -1, stream=s), dev)
        res["graph"] = {"ours_ms": ours_g}
        for name, fn in (("standard_attention", standard), ("sdpa", sdpa)):
            if "ms" in res[name]:
                theirs = graph_ms(lambda s: fn(), dev)
                res["graph"][name] = {"ms": theirs, "speedup": theirs / ours_g}
    except (RuntimeError, torch.cuda.OutOfMemoryError) as exc:
        res["graph"] = {"unavailable": str(exc).splitlines()[0][:200]}
    res["what"] = ("informative: standard = the pages' eager (q @ k^T * scale).softmax(-1) @ v (torch, cuBLAS); "
                   "sdpa = torch scaled_dot_product_attention (library kernel); speedup = their ms / ours; "
                   "graph = 20 calls per CUDA graph, replayed (no host launch cost)")
    return res


def oracle_rows_tflops(w: W.Workload, qkv, rows_per_head: int, heads=None):
    """Time the fp64 oracle on `rows_per_head` sampled rows of each selected (b, h).

    Returns (TFLOP/s-equivalent, seconds, rows, threads).  The FLOP credited per
    row is the workload's average per row, 4 * N_k * D * block_fraction.
    """
    from oracle import attention_ref
    rows = W.sample_rows(w, count=rows_per_head)
    heads = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.H)]
    t0 = time.perf_counter()
    for b, h in heads:
        hk = h * w.h_kv // w.H   # the K/V head this query head reads
        q = (qkv.q[b:b + 1, :, h:h + 1].to(torch.float64) * qkv.q_descale).numpy()
        k = (qkv.k[b:b + 1, :, hk:hk + 1].to(torch.float64) * qkv.k_descale).numpy()
        v = (qkv.v[b:b + 1, :, hk:hk + 1].to(torch.float64) * qkv.v_descale).numpy()
        attention_ref(q, k, v, w.scale, w.causal, w.window_left, rows=rows)
    dt = time.perf_counter() - t0
    per_row = 4.0 * w.n_k * w.D * W.block_fraction(w.n_q, w.n_k, w.causal, w.window_left)
    n_rows = len(rows) * len(heads)
    return per_row * n_rows / dt / 1e12, dt, n_rows, blas_threads()


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle, timed on this host's cores."""
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    qkv = inputs.make_qkv(w.B, w.n_q, w.n_k, w.H, w.D, w.dtype, seeds=w.seeds, h_kv=w.h_kv)
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    rows_per_step = args.reference_rows
    for i in range(args.warmup):
        oracle_rows_tflops(w, qkv, rows_per_step, heads=[heads[i % len(heads)]])
    total_t = 0.0
    total_rows = 0
    t_all = time.perf_counter()
    for i in range(args.steps):
        _, dt, n, threads = oracle_rows_tflops(w, qkv, rows_per_step, heads=[heads[i % len(heads)]])
        total_t += dt
        total_rows += n
    wall = time.perf_counter() - t_all
    per_row = 4.0 * w.n_k * w.D * W.block_fraction(w.n_q, w.n_k, w.causal, w.window_left)
    value = per_row * total_rows / total_t / 1e12
    sample = (f"each step: fp64 oracle on {rows_per_step} sampled query rows of one (batch, head), "
              f"cycling over the {len(heads)} heads; {args.steps} steps took {wall:.1f} s")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "desc": w.desc, "rows_per_step": rows_per_step,
                   "ms_per_step_note": "measured: one sampled step (the rows above), not a full forward"},
        # one full forward of the workload at the sampled throughput (an extrapolation)
        "full_forward_ms_extrapolated": W.flops(w) / (value * 1e12) * 1e3,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


MUFU_EXP_PER_CLK_PER_SM = 16   # ex2.approx results per clock per SM (B200 microbenchmark)
# configurations measured beside the headline in every run (the other configurations
# the target names), with the oracle rows per (batch, head) timed for each
EXTRA_CONFIGS = [("pr1_b1h8n512d64_fp16", 512), ("b2h8n2048d64_fp16", 64),
                 ("swa4096_b1h32n32768d128_bf16", 16), ("fp8_causal_b2h16n16384d128", 16)]


def binding_roofline(w: W.Workload, sms: int, sm_max_mhz: float):
    """(bound, peak TF/s, source) for a workload: the lower of the tensor-core
    peak (measured bf16 burst; x2 for e4m3) and the exponential unit's: one
    ex2 per score, MUFU_EXP_PER_CLK_PER_SM per SM per clock, 4 * D counted
    FLOP per score (2 D for Q.K, 2 D for P.V), at the maximum SM clock."""
    tensor, src, _ = measured_peaks(w.dtype)
    mhz = sm_max_mhz or 1965.0
    exp_peak = MUFU_EXP_PER_CLK_PER_SM * 4.0 * w.D * sms * mhz * 1e6 / 1e12
    if exp_peak < tensor:
        return "exp", exp_peak, (f"MUFU ex2 {MUFU_EXP_PER_CLK_PER_SM}/clk/SM x 4*D={4 * w.D} flop per score x "
                                 f"{sms} SMs x {mhz:.0f} MHz")
    return "tensor", tensor, f"{src} bf16 burst" + (" x2 for fp8" if w.dtype == "e4m3" else "")


def clock_normalised(value, clocks):
    """The value scaled to the maximum SM clock (value x max MHz / median MHz under load)."""
    if not clocks or not clocks.get("sm_mhz") or not clocks.get("sm_max_mhz"):
        return None
    return value * clocks["sm_max_mhz"] / clocks["sm_mhz"]


def timed(step, steps, dev, stream, local, barrier=lambda: None):
    """CUDA-event milliseconds of `steps` calls of step() on `stream`, with the
    SM clocks sampled while they run."""
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    return e0.elapsed_time(e1), sampler.stop()


def make_step(w: W.Workload, qkv, q, k, v, out, lse, stream, splits, mask):
    from exact_attention_136_b200 import forward, forward_fp8

    def step():
        if w.dtype == "e4m3":
            forward_fp8(q, k, v, qkv.q_descale, qkv.k_descale, qkv.v_descale, w.scale, w.causal, w.window_left,
                        out=out, lse=lse, stream=stream, num_splits=splits, attn_mask=mask)
        else:
            forward(q, k, v, w.scale, w.causal, w.window_left, out=out, lse=lse, stream=stream, num_splits=splits,
                    attn_mask=mask)
    return step


def device_tensors(w: W.Workload, seeds, dev):
    qkv = inputs.make_qkv(w.B, w.n_q, w.n_k, w.H, w.D, w.dtype, seeds=seeds, h_kv=w.h_kv)
    q, k, v = (t.pin_memory().to(dev) for t in (qkv.q, qkv.k, qkv.v))
    out_dtype = torch.float16 if w.dtype == "fp16" else torch.bfloat16
    out = torch.empty((w.B, w.n_q, w.H, w.D), dtype=out_dtype, device=dev)
    lse = torch.empty((w.B, w.H, w.n_q), dtype=torch.float32, device=dev)
    return qkv, q, k, v, out, lse


def measure_config(name, cpu_rows, dev, stream, local, sms, with_cpu):
    """One more configuration: launches timed for about 0.1 s after 5 warm-ups,
    its binding roofline, clocks, and the oracle on sampled rows."""
    from exact_attention_136_b200 import device_status
    w = W.WORKLOADS[name]
    qkv, q, k, v, out, lse = device_tensors(w, w.seeds, dev)
    step = make_step(w, qkv, q, k, v, out, lse, stream, w.splits, None)
    for _ in range(5):
        step()
    ms_try, _ = timed(step, 3, dev, stream, local)
    steps = int(min(2000, max(10, math.ceil(100.0 / max(ms_try / 3, 1e-3)))))
    ms, clocks = timed(step, steps, dev, stream, local)
    rc, flags = device_status(device=dev)
    if rc != 0:
        raise RuntimeError(f"{name}: device status {rc} flags {flags}")
    if not bool(torch.isfinite(out).all()):
        raise RuntimeError(f"{name}: non-finite output")
    ms_launch = ms / steps
    tf = W.flops(w) / (ms_launch / 1e3) / 1e12
    bound, peak, src = binding_roofline(w, sms, (clocks or {}).get("sm_max_mhz"))
    entry = {"desc": w.desc, "dtype": w.dtype, "launches": steps, "ms_per_launch": ms_launch,
             "us_per_launch": ms_launch * 1e3, "tflops": tf, "flop_per_launch": W.flops(w),
             "roofline": {"bound": bound, "peak": peak, "frac": tf / peak, "peak_source": src},
             "pct_of_nominal_dense_peak": 100.0 * tf / NOMINAL_TFLOPS[w.dtype],
             "clocks": clocks, "tflops_clock_normalised": clock_normalised(tf, clocks)}
    ctx = standard_attention_context(w, q, k, v, ms_launch, dev, stream)
    if ctx is not None:
        entry["vs_standard_attention"] = ctx
    if with_cpu:
        ctf, cdt, n_rows, threads = oracle_rows_tflops(w, qkv, cpu_rows)
        entry["cpu_oracle"] = {"tflops": ctf, "seconds": cdt, "rows": n_rows, "cores": threads,
                               "rows_per_head": min(cpu_rows, w.n_q)}
    del q, k, v, out, lse
    return entry


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.HEADLINE, choices=W.ORDER)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--splits", type=int, default=None, help="override the workload's key-range slices")
    ap.add_argument("--cpu-rows", type=int, default=128, help="oracle rows per (batch, head) for cpu_baseline")
    ap.add_argument("--reference-rows", type=int, default=256, help="oracle rows per step in --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling cases)")
    ap.add_argument("--backward", action="store_true", help="time the backward (fa_bwd) instead of the forward")
    ap.add_argument("--long-seconds", type=float, default=2.2,
                    help="also time the workload for at least this long (sustained figure; 0 = skip)")
    ap.add_argument("--no-extras", action="store_true", help="skip the other configurations")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_info()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    from exact_attention_136_b200 import _lib, device_status, forward_host

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    lib = _lib.lib()  # loud failure when the CUDA library is missing
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    w = W.WORKLOADS[args.workload]
    if args.batch is not None:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch, name=f"{w.name}@B{args.batch}")
    if args.backward:
        run_backward(args, w, world, rank, local, dev)
        return
    seeds = rank_seeds(w, rank)   # each rank: its own batch
    qkv, q, k, v, out, lse = device_tensors(w, seeds, dev)
    hq, hk, hv = qkv.q.pin_memory(), qkv.k.pin_memory(), qkv.v.pin_memory()
    out_dtype = out.dtype
    stream = torch.cuda.current_stream(dev)

    splits = w.splits if args.splits is None else args.splits
    mask_cpu = W.make_mask(w)
    mask = mask_cpu.to(dev) if mask_cpu is not None else None
    step = make_step(w, qkv, q, k, v, out, lse, stream, splits, mask)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    rc, flags = device_status(device=dev)
    if rc != 0:
        raise RuntimeError(f"device status {rc} flags {flags} after warm-up")

    ms, clocks = timed(step, args.steps, dev, stream, local, barrier)
    ms = max_over_ranks(ms, dev)
    rc, flags = device_status(device=dev)
    if rc != 0:
        raise RuntimeError(f"device status {rc} flags {flags} in the timed region")
    if not bool(torch.isfinite(out).all()):
        raise RuntimeError("non-finite output")

    flops = W.flops(w)
    ms_per_step = ms / args.steps
    value = world * flops * args.steps / (ms / 1e3) / 1e12
    per_launch_tflops = flops / (ms_per_step / 1e3) / 1e12

    # the same launches for a few seconds: what the kernel sustains under the power cap
    long_run = None
    if args.long_seconds > 0:
        n_long = int(math.ceil(args.long_seconds * 1e3 / ms_per_step))
        lms, lclocks = timed(step, n_long, dev, stream, local, barrier)
        lms = max_over_ranks(lms, dev)
        lval = world * flops * n_long / (lms / 1e3) / 1e12
        long_run = {"launches": n_long, "seconds": lms / 1e3, "ms_per_step": lms / n_long, "value": lval,
                    "clocks": lclocks, "value_clock_normalised": clock_normalised(lval, lclocks)}

    # end to end through the host-buffer entry point: H2D inputs, kernel, D2H out + lse, every step.
    # Three streams, each with its own device staging and pinned result buffers, take the steps in
    # turn (fa_fwd_host_async), so a step's copies in overlap the previous steps' forward and copies
    # out; grouped heads, split key ranges and masks go through pinned copies and the Python forward,
    # one step at a time.
    piped = w.h_kv == w.H and splits == 1 and mask is None
    n_pipe = 3 if piped else 1
    e2e_streams = [stream] + [torch.cuda.Stream(dev) for _ in range(n_pipe - 1)]
    stagings = [{"q": q, "k": k, "v": v, "out": out, "lse": lse}] + [
        {"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
         "out": torch.empty_like(out), "lse": torch.empty_like(lse)} for _ in range(n_pipe - 1)]
    hos = [torch.empty((w.B, w.n_q, w.H, w.D), dtype=out_dtype, pin_memory=True) for _ in range(n_pipe)]
    hls = [torch.empty((w.B, w.H, w.n_q), dtype=torch.float32, pin_memory=True) for _ in range(n_pipe)]
    desc = (qkv.q_descale, qkv.k_descale, qkv.v_descale)
    turn = [0]

    def e2e_step():
        i = turn[0] % n_pipe
        turn[0] += 1
        if piped:
            forward_host(hq, hk, hv, stagings[i], w.scale, w.causal, w.window_left, desc, hos[i], hls[i],
                         e2e_streams[i], synchronize=False)
        else:
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            step()
            hos[0].copy_(out, non_blocking=True)
            hls[0].copy_(lse, non_blocking=True)
            stream.synchronize()

    for _ in range(2 * n_pipe):
        e2e_step()
    barrier()
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s_ in e2e_streams[1:]:
        s_.wait_event(t0)
    for _ in range(args.e2e_steps):
        e2e_step()
    for s_ in e2e_streams[1:]:
        stream.wait_stream(s_)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ems = max_over_ranks(t0.elapsed_time(t1), dev)
    e2e_value = world * flops * args.e2e_steps / (ems / 1e3) / 1e12
    # every step computed the same forward: each stream's host result equals the device-timed run's
    ref_out = stagings[0]["out"].cpu()
    for i in range(n_pipe if piped else 0):
        if not torch.equal(hos[i], ref_out):
            raise RuntimeError(f"e2e: host result of stream {i} differs from the device forward")
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = hos[0].numel() * hos[0].element_size() + hls[0].numel() * hls[0].element_size()
    del stagings, e2e_streams

    peak, peak_src, sustained = measured_peaks(w.dtype)
    bound, bpeak, bsrc = binding_roofline(w, sms, (clocks or {}).get("sm_max_mhz"))
    traffic = recorded_traffic(w.name)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, dt, n_rows, threads = oracle_rows_tflops(w, qkv, args.cpu_rows)
        cpu = {"value": tf, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"fp64 oracle on {args.cpu_rows} sampled query rows of each of the {w.B * w.H} "
                         f"(batch, head) pairs ({n_rows} rows, {dt:.1f} s); FLOP credited per row = "
                         f"the workload's average 4*N_k*D*block_fraction"}
    del hq, hk, hv, hos, hls

    # the other configurations, one after another on this GPU (rank 0 of a single-GPU run)
    configs = None
    if rank == 0 and world == 1 and not args.no_extras and args.batch is None:
        del q, k, v, out, lse, step
        torch.cuda.empty_cache()
        configs = {w.name: {"desc": w.desc, "dtype": w.dtype, "ms_per_launch": ms_per_step,
                            "tflops": per_launch_tflops,
                            "roofline": {"bound": bound, "peak": bpeak, "frac": per_launch_tflops / bpeak,
                                         "peak_source": bsrc},
                            "pct_of_nominal_dense_peak": 100.0 * per_launch_tflops / NOMINAL_TFLOPS[w.dtype],
                            "clocks": clocks, "tflops_clock_normalised": clock_normalised(per_launch_tflops, clocks),
                            "note": "the headline measurement above"}}
        for name, rows in EXTRA_CONFIGS:
            if name != w.name:
                configs[name] = measure_config(name, rows, dev, stream, local, sms, not args.no_cpu_baseline)
                torch.cuda.empty_cache()

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "desc": w.desc, "B": w.B, "N_q": w.n_q, "N_k": w.n_k, "H": w.H,
                   "H_kv": w.h_kv, "splits": splits, "mask": w.mask or None, "D": w.D, "causal": w.causal,
                   "window_left": w.window_left, "scale": w.scale, "flop_per_step": flops,
                   "block_fraction": W.block_fraction(w.n_q, w.n_k, w.causal, w.window_left),
                   "l2": f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB vs {L2_BYTES / 1e6:.0f} MB), no flush",
                   "pct_of_nominal_dense_peak": 100.0 * per_launch_tflops / NOMINAL_TFLOPS[w.dtype],
                   "nominal_dense_peak_tflops": NOMINAL_TFLOPS[w.dtype],
                   "parallelism": f"replicas x{world} (independent batches per GPU)"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps,
                "api": "fa_fwd_host_async (pinned host buffers), 3 streams in turn: a step's copies in overlap "
                       "the previous steps' forward and copies out" if piped
                       else "pinned host copies + forward, one step at a time"},
        "roofline": {"bound": bound, "achieved": per_launch_tflops, "peak": bpeak, "unit": UNIT,
                     "frac": per_launch_tflops / bpeak, "traffic": traffic, "peak_source": bsrc,
                     "tensor_peak": peak, "tensor_peak_source": f"{peak_src} bf16 burst" +
                     (" x2 for fp8" if w.dtype == "e4m3" else ""), "peak_sustained": sustained},
        "value_clock_normalised": clock_normalised(value, clocks),
        "long_window": long_run,
        "configs": configs,
        "cpu_baseline": cpu,
        "clocks": clocks,
        "gpu_launches": args.steps,
        "kernel_hash": kernel_hash(),
    }
    print(json.dumps(line), flush=True)


def oracle_backward_tflops(w: W.Workload, qkv, dout):
    """The fp64 oracle's backward on one full (batch, head) of the workload
    (bounded sample: about 10-30 s for N = 8192); FLOP credited like the GPU's."""
    sys.path.insert(0, ROOT)
    from oracle import attention_backward_ref
    f = lambda t: t[:1, :, :1].double().numpy()
    t0 = time.perf_counter()
    attention_backward_ref(f(qkv.q), f(qkv.k), f(qkv.v), f(dout), w.scale, w.causal, w.window_left)
    dt = time.perf_counter() - t0
    flop = BWD_FLOP_RATIO * W.flops(w) / (w.B * w.H)
    return flop / dt / 1e12, dt, blas_threads()


def run_backward(args, w, world, rank, local, dev):
    from exact_attention_136_b200 import backward, device_status, forward

    if w.dtype == "e4m3" or w.h_kv != w.H or w.mask or w.splits != 1:
        raise SystemExit("--backward takes fp16 / bf16 workloads with K/V heads = query heads, no mask or split")
    seeds = rank_seeds(w, rank)
    qkv = inputs.make_qkv(w.B, w.n_q, w.n_k, w.H, w.D, w.dtype, seeds=seeds)
    g = inputs.make_qkv(w.B, w.n_q, w.n_q, w.H, w.D, w.dtype, seeds=tuple(x + 17 for x in seeds)).q
    host = {n: t.pin_memory() for n, t in (("q", qkv.q), ("k", qkv.k), ("v", qkv.v), ("dout", g))}
    q, k, v, dout = (host[n].to(dev) for n in ("q", "k", "v", "dout"))
    stream = torch.cuda.current_stream(dev)
    out, lse = forward(q, k, v, w.scale, w.causal, w.window_left, stream=stream)
    host["out"], host["lse"] = out.cpu().pin_memory(), lse.cpu().pin_memory()

    def step():
        return backward(q, k, v, out, lse, dout, w.scale, w.causal, w.window_left, stream=stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        grads = step()
    torch.cuda.synchronize(dev)
    rc, flags = device_status(device=dev)
    if rc != 0:
        raise RuntimeError(f"device status {rc} flags {flags} after warm-up")
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(args.steps):
        grads = step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    rc, flags = device_status(device=dev)
    if rc != 0:
        raise RuntimeError(f"device status {rc} flags {flags} in the timed region")
    if not all(bool(torch.isfinite(t).all()) for t in grads):
        raise RuntimeError("non-finite gradient")
    flops = BWD_FLOP_RATIO * W.flops(w)
    ms_per_step = ms / args.steps
    value = world * flops * args.steps / (ms / 1e3) / 1e12
    per_step_tflops = flops / (ms_per_step / 1e3) / 1e12

    # end to end: inputs (q, k, v, out, lse, dout) from pinned host memory,
    # the backward, and dq, dk, dv back to pinned host memory
    hg = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (q, k, v)]

    def e2e_step():
        for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("dout", dout)):
            t.copy_(host[name], non_blocking=True)
        for hdst, dsrc in zip(hg, step()):
            hdst.copy_(dsrc, non_blocking=True)
        stream.synchronize()

    for _ in range(2):
        e2e_step()
    barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ems = max_over_ranks(t0.elapsed_time(t1), dev)
    e2e_value = world * flops * args.e2e_steps / (ems / 1e3) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in hg)

    peak, peak_src, sustained = measured_peaks(w.dtype)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, dt, threads = oracle_backward_tflops(w, qkv, g)
        cpu = {"value": tf, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"fp64 oracle backward on one full (batch, head) of the {w.B * w.H} ({dt:.1f} s); "
                         f"FLOP credited as 2.5x the forward's per head"}
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v, out, dout))
    line = {
        "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": "bwd_" + w.name, "desc": "backward of " + w.desc, "B": w.B, "N_q": w.n_q,
                   "N_k": w.n_k, "H": w.H, "D": w.D, "causal": w.causal, "window_left": w.window_left,
                   "scale": w.scale, "flop_per_step": flops,
                   "block_fraction": W.block_fraction(w.n_q, w.n_k, w.causal, w.window_left),
                   "l2": f"inputs larger than L2 ({in_bytes / 1e6:.0f} MB vs {L2_BYTES / 1e6:.0f} MB), no flush",
                   "pct_of_nominal_dense_peak": 100.0 * per_step_tflops / NOMINAL_TFLOPS[w.dtype],
                   "nominal_dense_peak_tflops": NOMINAL_TFLOPS[w.dtype],
                   "parallelism": f"replicas x{world} (independent batches per GPU)"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps, "api": "pinned host copies + backward"},
        "roofline": {"bound": "tensor", "achieved": per_step_tflops, "peak": peak, "unit": UNIT,
                     "frac": per_step_tflops / peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16 burst", "peak_sustained": sustained,
                     "note": "achieved over the whole step (three kernels: row term, dK/dV, dQ)"},
        "cpu_baseline": cpu,
        "clocks": clocks,
        "gpu_launches": 3 * args.steps,   # row term, dK/dV kernel, dQ kernel per step
        "kernel_hash": kernel_hash(),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
