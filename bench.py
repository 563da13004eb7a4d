"""Benchmark of one decode step of the paged-KV hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one pass of the whole hot path over one batch: the copy-on-write
block copies (when the workload has shared blocks), the write of each
sequence's new token into its slot, and paged decode attention (partition and
reduce kernels).  The default workload is the Llama-3-8B-shaped GQA decode
(256 sequences, 32 query / 8 KV heads, head dim 128, bf16, log-normal context
lengths with median 1024 clipped to [128, 4096]).

The metric is KV-read GB/s: the algorithmic K+V bytes a decode call reads
(sum_b L_b * Hkv * 2 * D * element bytes) per step, divided by the step time,
summed over ranks.  Rank 0 prints one JSON line.  ``--impl reference`` times the
fp64 CPU oracle on the host cores instead (bounded sample of the same
workload) and prints the same kind of line.

Multi-GPU (torchrun): every rank decodes its own batch of the same shape
(seed offset by rank); there is no exchange on the data path; the step time is
the maximum over ranks.

``--workload llama3_8b_prefill`` measures paged chunked prefill instead: a step
writes the chunk tokens' K/V into their slots (pa_reshape_and_cache) and runs
pa_prefill (16 sequences, 512-token chunks after cached prefixes of 0..1536
tokens, 32 query / 8 KV heads, head dim 128, bf16); the metric is attention
TFLOP/s over the causally visible (query, key) pairs.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from paged_kv_cache_464_b200 import inputs  # noqa: E402

METRIC = "paged decode attention: KV-read GB/s (% of B200 HBM peak), seqs/s"
PREFILL_METRIC = "paged chunked-prefill attention: TFLOP/s (% of B200 bf16 tensor peak)"
FALLBACK_BF16_TFLOPS = 1590.0
DEFAULT_WORKLOAD = "llama3_8b_gqa"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def rank_seed(cfg: inputs.DecodeConfig, rank: int) -> int:
    """Each rank draws its own batch of the workload's shape."""
    return cfg.seed + 7919 * rank


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure (a prefill step is well under a second)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def profiled_traffic(workload: str, kernel: str = "pa_decode"):
    """DRAM bytes (read + write) per call of `kernel` from the committed ncu summary,
    or None when there is none or the kernel sources changed since it was taken."""
    from paged_kv_cache_464_b200 import build
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("source_sha256") != build.source_digest():
        return None
    return d.get("dram_bytes_per_call")


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms in a background process."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []   # (t, sm_mhz, max_mhz, reasons)
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            reasons = [n for n, v in zip(names, parts[5:9]) if v.lower() == "active"]
            self.samples.append((time.time(), sm, mx, reasons))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        window = [s for s in self.samples if t0 <= s[0] <= t1]
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({r for s in window for r in s[3]})
        return {"sm_mhz": statistics.median(s[1] for s in window), "sm_max_mhz": max(s[2] for s in window),
                "reasons": reasons, "samples": len(window)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def all_reduce_max(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_reduce_sum(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ timing helpers
def percentile(xs, q: float) -> float:
    """The q-th percentile of xs (linear interpolation between order statistics)."""
    ys = sorted(xs)
    if not ys:
        return float("nan")
    k = (len(ys) - 1) * q / 100.0
    lo = int(math.floor(k))
    hi = min(lo + 1, len(ys) - 1)
    return ys[lo] + (ys[hi] - ys[lo]) * (k - lo)


def spread_line(ms, work, peak, unit, scale, what):
    """Mean / median / p10 / p90 of per-call times and the work rate at the median."""
    med = statistics.median(ms)
    rate = work / (med * 1e-3) / scale
    return {"calls": len(ms), "ms_mean": round(statistics.mean(ms), 5), "ms_median": round(med, 5),
            "ms_p10": round(percentile(ms, 10), 5), "ms_p90": round(percentile(ms, 90), 5),
            "achieved_at_median": round(rate, 2), "unit": unit, "frac_at_median": round(rate / peak, 4),
            "what": what}


def back_to_back(call, n, stream):
    """Mean duration (ms) of ``call`` over n calls in a row, events at both ends only."""
    for _ in range(3):
        call()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def l2_flushed_calls(pre, call, n, stream, device):
    """Per-call times of ``call`` (events on its stream), each call preceded by
    ``pre`` and by a 256 MiB write (2x the L2) outside the events."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        pre()
        flush.fill_(i & 0xff)
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    del flush
    return [a.elapsed_time(b) for a, b in ev]


def stream_read_probe(device, nbytes: int = 2 << 30, reps: int = 20):
    """Read-only bandwidth of the library's plain streaming-read kernel
    (pa_stream_read) over a buffer 16x the L2, median of ``reps`` timed reads."""
    from paged_kv_cache_464_b200 import capi
    buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
    buf.fill_(1)
    sink = torch.zeros(1, dtype=torch.int64, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(3):
        capi.stream_read(buf, sink)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        a.record(stream)
        capi.stream_read(buf, sink)
        b.record(stream)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    del buf
    med = statistics.median(ms)
    return {"kernel": "pa_stream_read (16-byte streaming loads, 8 CTAs x 256 threads per SM)",
            "bytes": nbytes, "ms_median": round(med, 5), "gbs_median": round(nbytes / (med * 1e-3) / 1e9, 1),
            "gbs_best": round(nbytes / (min(ms) * 1e-3) / 1e9, 1), "reps": reps}


# ------------------------------------------------------------------ our arm
class Step:
    """The device buffers of one workload and the step's calls through the C ABI."""

    def __init__(self, case: inputs.DecodeCase, device):
        from paged_kv_cache_464_b200 import capi
        self.pa = capi
        self.case = case
        c = case.cfg
        self.q = case.q.to(device)
        self.k = case.k_cache.to(device)
        self.v = case.v_cache.to(device)
        self.key = case.key.to(device)
        self.value = case.value.to(device)
        self.slots = case.slot_mapping.to(device)
        self.pairs = case.block_mapping.to(device)
        self.bt = case.block_tables.to(device)
        self.cl = case.context_lens.to(device)
        self.out = torch.empty_like(self.q)
        self.maxL = case.max_context_len
        self.P = c.partition_size
        ws = capi.decode_workspace_bytes(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, self.maxL, self.P)
        self.ws = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.has_pairs = case.block_mapping.numel() > 0
        self.fp8 = c.kv_dtype == "fp8_e4m3"
        if self.fp8:
            # 1-byte caches: quantise the whole pool once (setup, not timed)
            nb, bs, hkv, d = self.k.shape
            self.kv_scale = c.kv_scale
            k8 = torch.zeros((nb, bs, hkv, d), dtype=torch.uint8, device=device)
            v8 = torch.zeros_like(k8)
            slots = torch.arange(nb * bs, dtype=torch.int64, device=device)
            capi.reshape_and_cache_fp8(self.k.view(nb * bs, hkv, d), self.v.view(nb * bs, hkv, d), k8, v8, slots,
                                       self.kv_scale, self.kv_scale)
            torch.cuda.synchronize()
            self.k, self.v = k8, v8

    def launches(self, fused: bool) -> int:
        c = self.case.cfg
        P = self.pa.decode_partition_size(c.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, self.maxL, self.P)
        split = math.ceil(self.maxL / P) > 1
        return (1 if self.has_pairs else 0) + (0 if fused and not self.fp8 else 1) + 1 + (1 if split else 0)

    # fused step: copies, then the new-token write and decode in one launch (pa_decode_append);
    # 1-byte caches: copies, the quantising new-token write, then pa_decode_fp8
    def pre(self):
        if self.has_pairs:
            self.pa.copy_blocks(self.k, self.v, self.pairs)
        if self.fp8:
            self.pa.reshape_and_cache_fp8(self.key, self.value, self.k, self.v, self.slots, self.kv_scale,
                                          self.kv_scale)

    def decode(self):
        if self.fp8:
            self.pa.decode_fp8(self.q, self.k, self.v, self.kv_scale, self.kv_scale, self.bt, self.cl,
                               self.case.scale, out=self.out, max_context_len=self.maxL, partition_size=self.P,
                               workspace=self.ws)
            return
        self.pa.decode_append(self.q, self.key, self.value, self.k, self.v, self.bt, self.cl, self.case.scale,
                              out=self.out, max_context_len=self.maxL, partition_size=self.P, workspace=self.ws)

    def __call__(self):
        self.pre()
        self.decode()

    def raw_calls(self, t, out, stream):
        """The step as (C function, argument tuple) pairs over the tensors ``t``
        (name -> device tensor: q, key, value, slots, pairs, bt, cl) and ``out``,
        arguments marshalled once, for a loop that calls the C ABI directly."""
        r, c, case = self.pa.raw, self.case.cfg, self.case
        nb, bs, hkv, d = self.k.shape
        s = stream.cuda_stream
        ws, wsb = self.ws.data_ptr(), self.ws.numel()
        S, hq, mbs = c.num_seqs, c.num_heads, t["bt"].shape[1]
        calls = []
        if self.has_pairs:
            calls.append((r.pa_copy_blocks, (self.k.data_ptr(), self.v.data_ptr(), t["pairs"].data_ptr(),
                                             t["pairs"].shape[0], nb, bs, hkv, d, self.pa.DTYPE_CODE[self.q.dtype]
                                             if not self.fp8 else self.pa.FP8, s)))
        if self.fp8:
            qd = self.pa.DTYPE_CODE[self.q.dtype]
            calls.append((r.pa_reshape_and_cache_fp8, (t["key"].data_ptr(), t["value"].data_ptr(), self.k.data_ptr(),
                                                       self.v.data_ptr(), t["slots"].data_ptr(), t["key"].shape[0], nb,
                                                       bs, hkv, d, qd, self.kv_scale, self.kv_scale, s)))
            calls.append((r.pa_decode_fp8, (out.data_ptr(), t["q"].data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                                            self.kv_scale, self.kv_scale, t["bt"].data_ptr(), mbs, t["cl"].data_ptr(),
                                            S, hq, self.maxL, case.scale, self.P, ws, wsb, nb, bs, hkv, d, qd, s)))
        else:
            dt = self.pa.DTYPE_CODE[self.q.dtype]
            calls.append((r.pa_decode_append, (out.data_ptr(), t["q"].data_ptr(), t["key"].data_ptr(),
                                               t["value"].data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                                               t["bt"].data_ptr(), mbs, t["cl"].data_ptr(), S, hq, self.maxL,
                                               case.scale, self.P, ws, wsb, nb, bs, hkv, d, dt, s)))
        return calls

    # the same step as three separate calls (pa_copy_blocks, pa_reshape_and_cache, pa_decode)
    def separate(self):
        if self.fp8:
            self()
            return
        if self.has_pairs:
            self.pa.copy_blocks(self.k, self.v, self.pairs)
        self.pa.reshape_and_cache(self.key, self.value, self.k, self.v, self.slots)
        self.pa.decode(self.q, self.k, self.v, self.bt, self.cl, self.case.scale, out=self.out,
                       max_context_len=self.maxL, partition_size=self.P, workspace=self.ws)


def run_ours(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    sampler = ClockSampler(local).start()   # started early: nvidia-smi takes a moment to report
    cfg = inputs.CONFIGS[args.workload]
    case = inputs.make_case(cfg, seed=rank_seed(cfg, rank), with_post=False)
    step = Step(case, device)
    kv_bytes = case.kv_bytes()
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- timed region: exactly K steps, events only at its two ends (an event
    # between launches would stop the next kernel from being scheduled early)
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start.record(stream)
    for _ in range(args.steps):
        step()
    t_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = t_start.elapsed_time(t_stop)

    # ---- roofline pass: the same K steps with the decode launches bracketed by
    # events on the launching stream, for the kernel's own average duration
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        step.pre()
        ev_dec[i][0].record(stream)
        step.decode()
        ev_dec[i][1].record(stream)
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(b) for a, b in ev_dec]

    # ---- the decode call alone, K calls back to back with events only at the
    # two ends (launches overlap as in the step): the kernel's steady-state duration
    loop_ms = back_to_back(step.decode, args.steps, stream)

    # ---- the same calls with L2 flushed before each (a 256 MiB write between
    # steps, outside the events): shows the figures do not come from L2 reuse
    flushed_ms = l2_flushed_calls(step.pre, step.decode, min(args.steps, 200), stream, device)

    # the same K steps as three separate calls, for comparison
    for _ in range(args.warmup):
        step.separate()
    s_start, s_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    s_start.record(stream)
    for _ in range(args.steps):
        step.separate()
    s_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    sep_ms = s_start.elapsed_time(s_stop)

    # keep the GPU under the same load long enough for the clock sampler
    soak_until = wall0 + 2.5
    while time.time() < soak_until:
        for _ in range(50):
            step()
        torch.cuda.synchronize()
    wall_soak = time.time()
    sampler.stop()

    # ---- read-only bandwidth of a plain streaming-read kernel (context for the fraction)
    read_probe = stream_read_probe(device)

    # ---- end to end through the public API from pinned host buffers
    e2e = run_e2e(case, step, args.steps, args.warmup, device)

    max_ms = all_reduce_max(elapsed_ms, world, device)
    sep_max_ms = all_reduce_max(sep_ms, world, device)
    total_bytes = all_reduce_sum(float(kv_bytes), world, device)
    total_seqs = all_reduce_sum(float(cfg.num_seqs), world, device)
    e2e_ms = all_reduce_max(e2e["ms"], world, device)

    if rank != 0:
        return None
    ms_per_step = max_ms / args.steps
    value = total_bytes * args.steps / (max_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    achieved = kv_bytes / (loop_ms * 1e-3) / 1e9
    clocks = sampler.summary(wall0, wall_soak)
    traffic = profiled_traffic(args.workload)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8_e4m3 KV (f16 tensor-core math), bf16 q/out" if step.fp8 else cfg.dtype,
        "data": "synthetic (seeded N(0,1) Q/K/V, shuffled block pool)",
        "config": {
            "workload": cfg.name,
            "description": cfg.description,
            "num_seqs_per_gpu": cfg.num_seqs,
            "num_heads": cfg.num_heads,
            "num_kv_heads": cfg.num_kv_heads,
            "head_dim": cfg.head_dim,
            "block_size": cfg.block_size,
            "sum_context_len": int(case.context_lens.sum()),
            "kv_bytes_per_step_per_gpu": kv_bytes,
            "partition_size": step.pa.decode_partition_size(cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads,
                                                            cfg.head_dim, step.maxL, step.P),
            "step": ("pa_copy_blocks + " if step.has_pairs else "") + (
                "pa_reshape_and_cache_fp8 + pa_decode_fp8" if step.fp8 else
                "pa_decode_append (new-token write + decode)"),
            "kv_cache": "fp8_e4m3, scale %g" % cfg.kv_scale if step.fp8 else cfg.dtype,
            "l2": f"inputs larger than L2: {kv_bytes / 2**20:.0f} MiB of KV per step vs 126 MiB L2, no flush",
            "parallelism": f"replicas x{world}, no data-path collective",
        },
        "seqs_per_s": round(total_seqs * args.steps / (max_ms * 1e-3), 1),
        "step_separate_calls": {
            "calls": ("pa_copy_blocks + " if step.has_pairs else "") + (
                "pa_reshape_and_cache_fp8 + pa_decode_fp8" if step.fp8 else "pa_reshape_and_cache + pa_decode"),
            "value": round(total_bytes * args.steps / (sep_max_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "ms_per_step": round(sep_max_ms / args.steps, 5)},
        "pct_hbm_peak": round(100.0 * value / world / peak, 2),
        "roofline": {
            "kernel": ("pa_decode_fp8" if step.fp8 else "pa_decode_append") + " (partition + reduce launches)",
            "bound": "hbm",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback 6.65 TB/s",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "decode_ms_mean": round(loop_ms, 5),
            "decode_timing": f"{args.steps} decode calls back to back, events at both ends only",
            "frac_of_read_probe": round(achieved / read_probe["gbs_median"], 4),
            "per_call_events": spread_line(dec_ms, kv_bytes, peak, "GB/s", 1e9,
                                           "each call between two events (no overlap with its neighbours)"),
            "l2_flushed": spread_line(flushed_ms, kv_bytes, peak, "GB/s", 1e9,
                                      "the same calls, each after a 256 MiB write that evicts L2"),
            "read_probe": read_probe,
        },
        "e2e": {"value": round(total_bytes * args.steps / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": round(e2e_ms / args.steps, 5),
                "host_us_per_step": e2e["host_us"],
                "frac_of_value": round(max_ms / e2e_ms, 4),
                "path": e2e["path"]},
        "gpu_launches": step.launches(fused=True) * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, budget_s=args.cpu_budget)
    return line


# ------------------------------------------------------------------ chunked prefill
class PrefillStep:
    """Device buffers of a chunked-prefill batch; a step writes the chunk tokens'
    K/V rows into their slots and runs paged prefill attention."""

    def __init__(self, case: inputs.PrefillCase, device):
        from paged_kv_cache_464_b200 import capi
        self.pa = capi
        self.case = case
        NB, bs, Hkv, D = case.k_cache.shape
        self.slots_host = chunk_slots(case)
        self.key_host = case.k_cache.view(NB * bs, Hkv, D)[self.slots_host].contiguous()
        self.value_host = case.v_cache.view(NB * bs, Hkv, D)[self.slots_host].contiguous()
        self.q = case.q.to(device)
        self.kc, self.vc = case.k_cache.to(device), case.v_cache.to(device)
        self.bt, self.cl = case.block_tables.to(device), case.context_lens.to(device)
        self.qsl = case.query_start_loc.to(device)
        self.key, self.value = self.key_host.to(device), self.value_host.to(device)
        self.slots = self.slots_host.to(device)
        self.out = torch.empty_like(self.q)
        self.max_query_len = case.max_query_len

    def write(self):
        self.pa.reshape_and_cache(self.key, self.value, self.kc, self.vc, self.slots)

    def attend(self):
        self.pa.prefill(self.q, self.kc, self.vc, self.bt, self.cl, self.qsl, self.case.scale, self.out,
                        max_query_len=self.max_query_len)

    def __call__(self):
        self.write()
        self.attend()

    def raw_calls(self, t, out, stream):
        """The step as (C function, argument tuple) pairs over the tensors ``t``
        (q, key, value, slots, bt, cl, qsl) and ``out``; see Step.raw_calls."""
        r, c = self.pa.raw, self.case.cfg
        nb, bs, hkv, d = self.kc.shape
        dt = self.pa.DTYPE_CODE[self.q.dtype]
        s = stream.cuda_stream
        return [(r.pa_reshape_and_cache, (t["key"].data_ptr(), t["value"].data_ptr(), self.kc.data_ptr(),
                                          self.vc.data_ptr(), t["slots"].data_ptr(), t["key"].shape[0], nb, bs, hkv,
                                          d, dt, s)),
                (r.pa_prefill, (out.data_ptr(), t["q"].data_ptr(), self.kc.data_ptr(), self.vc.data_ptr(),
                                t["bt"].data_ptr(), t["bt"].shape[1], t["cl"].data_ptr(), t["qsl"].data_ptr(),
                                c.num_seqs, c.num_heads, self.max_query_len, self.case.scale, nb, bs, hkv, d, dt, s))]


def chunk_slots(case: inputs.PrefillCase) -> torch.Tensor:
    """Slots of every chunk token (positions L - n .. L - 1 of each sequence), in query order."""
    bs = case.k_cache.shape[1]
    out = []
    for b in range(case.cfg.num_seqs):
        L = int(case.context_lens[b])
        n = int(case.query_start_loc[b + 1] - case.query_start_loc[b])
        pos = torch.arange(L - n, L)
        out.append(case.block_tables[b, pos // bs].to(torch.int64) * bs + pos % bs)
    return torch.cat(out) if out else torch.zeros(0, dtype=torch.int64)


def run_prefill(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    sampler = ClockSampler(local).start()
    cfg = inputs.PREFILL_CONFIGS[args.workload]
    case = inputs.make_prefill_case(cfg, seed=rank_seed(cfg, rank))
    step = PrefillStep(case, device)
    flops = case.flops()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start.record(stream)
    for _ in range(args.steps):
        step()
    t_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    elapsed_ms = t_start.elapsed_time(t_stop)

    # roofline pass: the attention launch bracketed by events on its stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        step.write()
        ev[i][0].record(stream)
        step.attend()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    att_ms = [a.elapsed_time(b) for a, b in ev]
    flushed_ms = l2_flushed_calls(step.write, step.attend, min(args.steps, 200), stream, device)
    loop_ms = back_to_back(step.attend, args.steps, stream)

    soak_until = wall0 + 2.5
    while time.time() < soak_until:
        for _ in range(20):
            step()
        torch.cuda.synchronize()
    wall_soak = time.time()
    sampler.stop()

    e2e = run_e2e_prefill(step, args.steps, args.warmup)
    max_ms = all_reduce_max(elapsed_ms, world, device)
    total_flops = all_reduce_sum(float(flops), world, device)
    e2e_ms = all_reduce_max(e2e["ms"], world, device)
    if rank != 0:
        return None
    value = total_flops * args.steps / (max_ms * 1e-3) / 1e12
    peak, peak_kind = measured_tensor_peak()
    achieved = flops / (loop_ms * 1e-3) / 1e12
    line = {
        "metric": PREFILL_METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": cfg.dtype,
        "data": "synthetic (seeded N(0,1) Q/K/V, shuffled block pool)",
        "config": {
            "workload": cfg.name,
            "description": cfg.description,
            "num_seqs_per_gpu": case.cfg.num_seqs,
            "num_heads": cfg.num_heads,
            "num_kv_heads": cfg.num_kv_heads,
            "head_dim": cfg.head_dim,
            "block_size": cfg.block_size,
            "query_tokens_per_step": case.num_tokens,
            "context_lens": case.context_lens.tolist(),
            "flops_per_step_per_gpu": flops,
            "flops_rule": "4 * Hq * D per causally visible (query, key) pair (QK^T and PV multiply-adds)",
            "step": "pa_reshape_and_cache (chunk K/V) + pa_prefill",
            "l2": "inputs larger than L2: q, out, chunk K/V and the attended KV of a step total "
                  f"{(2 * step.q.numel() * 2 + 2 * step.key.numel() * 2 + case.kv_bytes_attended()) / 2**20:.0f} MiB "
                  "vs 126 MiB L2, no flush",
            "parallelism": f"replicas x{world}, no data-path collective",
        },
        "pct_tensor_peak": round(100.0 * value / world / peak, 2),
        "roofline": {
            "kernel": "pa_prefill",
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_kind": "measured dense bf16 burst (MEASURED_PEAKS.json bf16_tflops)" if peak_kind == "measured"
            else "fallback 1.59 PFLOP/s",
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "traffic": profiled_traffic(args.workload, kernel="pa_prefill"),
            "prefill_ms_mean": round(loop_ms, 5),
            "prefill_timing": f"{args.steps} pa_prefill calls back to back, events at both ends only",
            "per_call_events": spread_line(att_ms, flops, peak, "TFLOP/s", 1e12,
                                           "each call between two events, after the step's K/V write"),
            "l2_flushed": spread_line(flushed_ms, flops, peak, "TFLOP/s", 1e12,
                                      "the same calls, each after a 256 MiB write that evicts L2"),
        },
        "e2e": {"value": round(total_flops * args.steps / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": round(e2e_ms / args.steps, 5),
                "host_us_per_step": e2e["host_us"],
                "frac_of_value": round(max_ms / e2e_ms, 4),
                "path": e2e["path"]},
        "gpu_launches": 2 * args.steps,
        "clocks": sampler.summary(wall0, wall_soak),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(case, budget_s=args.cpu_budget)
    return line


def run_e2e_prefill(step: PrefillStep, steps, warmup):
    """Per step: q, the chunk K/V rows, slots and tables host->device from pinned
    memory, the step through the C ABI, out device->host."""
    case = step.case
    host = {"q": case.q, "key": step.key_host, "value": step.value_host, "slots": step.slots_host,
            "bt": case.block_tables, "cl": case.context_lens, "qsl": case.query_start_loc}
    return pipelined_e2e(step, host, step.out, steps, warmup)


def _oracle_prefill(o, case):
    return o.paged_prefill(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                           case.query_start_loc, case.scale)


def _prefill_sample(case, budget_s):
    """A bounded sample: the first sequences whose oracle run fits the budget (calibrated on one)."""
    import oracle
    o = oracle.get()
    one = inputs.prefill_subcase(case, [0])
    t = time.perf_counter()
    _oracle_prefill(o, one)
    per_flop = (time.perf_counter() - t) / max(1, one.flops())
    n, fl = 0, 0
    while n < case.cfg.num_seqs:
        f = inputs.prefill_subcase(case, [n]).flops()
        if n > 0 and (fl + f) * per_flop > budget_s:
            break
        fl += f
        n += 1
    return o, inputs.prefill_subcase(case, list(range(n))), n


def cpu_baseline_prefill(case, budget_s: float = 20.0):
    o, sample, n = _prefill_sample(case, budget_s / 2)
    t = time.perf_counter()
    _oracle_prefill(o, sample)
    dt = time.perf_counter() - t
    return {"value": round(sample.flops() / dt / 1e12, 6), "unit": "TFLOP/s", "cores": o.num_threads,
            "kind": "oracle", "cpu": cpu_model(),
            "sample": f"first {n} of {case.cfg.num_seqs} sequences of the same workload (whole chunks), fp64, one run"}


def run_reference_prefill(args, world, rank):
    if rank != 0:
        return None
    cfg = inputs.PREFILL_CONFIGS[args.workload]
    case = inputs.make_prefill_case(cfg, seed=rank_seed(cfg, 0))
    o, sample, n = _prefill_sample(case, args.ref_budget / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        _oracle_prefill(o, sample)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_prefill(o, sample)
    el = time.perf_counter() - t0
    value = sample.flops() * args.steps / el / 1e12
    desc = f"first {n} of {cfg.num_seqs} sequences per step (fp64 paged prefill), {o.num_threads} threads"
    return {
        "metric": PREFILL_METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "description": cfg.description, "sample_seqs_per_step": n},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": o.num_threads, "kind": "oracle", "cpu": cpu_model(),
                         "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


class PackedInputs:
    """All of a step's input tensors in ONE pinned host buffer, and `sets`
    device buffers of the same layout (each tensor at a 256-byte-aligned
    offset), so a step's inputs move with one host->device copy; views into a
    device buffer feed the calls."""

    def __init__(self, tensors, device, sets=2):
        self.offsets, off = {}, 0
        for n, t in tensors.items():
            self.offsets[n] = off
            off += (t.numel() * t.element_size() + 255) // 256 * 256
        self.nbytes = off
        self.host = torch.zeros(off, dtype=torch.uint8).pin_memory()
        for n, t in tensors.items():
            o, nb = self.offsets[n], t.numel() * t.element_size()
            self.host[o:o + nb].copy_(t.contiguous().reshape(-1).view(torch.uint8))
        self.dev = [torch.empty(off, dtype=torch.uint8, device=device) for _ in range(sets)]
        self.views = []
        for buf in self.dev:
            v = {}
            for n, t in tensors.items():
                o, nb = self.offsets[n], t.numel() * t.element_size()
                v[n] = buf[o:o + nb].view(t.dtype).view(t.shape)
            self.views.append(v)


def pipelined_e2e(step, host, out_like, steps, warmup):
    """End to end through the C ABI: every step copies its inputs ``host``
    (name -> host tensor, packed into one pinned buffer) to the device in one
    copy, makes the step's C calls (arguments marshalled once, the call made
    directly, no per-call Python checks) and copies the output back into pinned
    host memory.  Three sets of device inputs and outputs rotate between steps,
    with one copy stream per direction, so that step k's input copy may run
    during the kernels of steps k-2 and k-1 and its output copy during those of
    step k+1 (as a serving loop would run them); every copy of every timed step
    lies inside the timed region.  Also reports the host time of issuing a step
    (a short burst timed with the GPU idle at its start)."""
    NSETS = 3
    compute = torch.cuda.current_stream()
    device = out_like.device
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    packed = PackedInputs(host, device, NSETS)
    outs = [torch.empty_like(out_like) for _ in range(NSETS)]
    out_host = [torch.empty(out_like.shape, dtype=out_like.dtype).pin_memory() for _ in range(NSETS)]
    calls = [step.raw_calls(packed.views[i], outs[i], compute) for i in range(NSETS)]
    loaded = [torch.cuda.Event() for _ in range(NSETS)]     # inputs of set i on the device
    consumed = [torch.cuda.Event() for _ in range(NSETS)]   # kernels that read set i (and write its output) done
    drained = [torch.cuda.Event() for _ in range(NSETS)]    # output of set i copied to the host

    def one(k):
        i = k % NSETS
        h2d_s.wait_event(consumed[i])                   # the step NSETS back is done with these inputs
        with torch.cuda.stream(h2d_s):
            packed.dev[i].copy_(packed.host, non_blocking=True)
        loaded[i].record(h2d_s)
        compute.wait_event(loaded[i])
        compute.wait_event(drained[i])                  # its output buffer has been read out
        for fn, a in calls[i]:
            rc = fn(*a)
            if rc != 0:
                raise RuntimeError(f"{fn.__name__}: status {rc}")
        consumed[i].record(compute)
        d2h_s.wait_event(consumed[i])
        with torch.cuda.stream(d2h_s):
            out_host[i].copy_(outs[i], non_blocking=True)
        drained[i].record(d2h_s)

    def loop(n):
        for i in range(NSETS):
            consumed[i].record(compute)
            drained[i].record(compute)
        h2d_s.wait_stream(compute)
        d2h_s.wait_stream(compute)
        for k in range(n):
            one(k)
        compute.wait_stream(h2d_s)
        compute.wait_stream(d2h_s)

    loop(max(NSETS, warmup))
    torch.cuda.synchronize()
    burst = min(steps, 32)
    t0 = time.perf_counter()
    loop(burst)
    host_us = (time.perf_counter() - t0) * 1e6 / burst
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(compute)
    loop(steps)
    b.record(compute)
    torch.cuda.synchronize()
    d2h = out_host[0].numel() * out_host[0].element_size()
    return {"ms": a.elapsed_time(b), "h2d": packed.nbytes, "d2h": d2h, "host_us": round(host_us, 2),
            "last_out_host": out_host[(steps - 1) % NSETS],
            "path": "one packed pinned->device copy, direct C-ABI calls, one device->pinned copy per step; "
                    "three buffer sets rotate so copies overlap the neighbouring steps' kernels"}


def run_e2e(case, step, steps, warmup, device):
    """Per step: inputs host->device from pinned memory, the step through the
    C ABI, the output device->host into pinned memory."""
    host = {"q": case.q, "key": case.key, "value": case.value, "slots": case.slot_mapping,
            "bt": case.block_tables, "cl": case.context_lens}
    if step.has_pairs:
        host["pairs"] = case.block_mapping
    return pipelined_e2e(step, host, step.out, steps, warmup)


# ------------------------------------------------------------------ oracle timings
def _sample_case(case: inputs.DecodeCase, n: int) -> inputs.DecodeCase:
    """The first n sequences of a case (same cache; copy pairs kept only for them)."""
    import dataclasses
    if n >= case.cfg.num_seqs:
        return case
    keep_pairs = case.block_mapping
    if keep_pairs.numel():
        rows = case.block_tables[:n].to(torch.int64)
        used = set(rows[rows >= 0].tolist())
        mask = torch.tensor([int(d) in used for d in keep_pairs[:, 1]], dtype=torch.bool)
        keep_pairs = keep_pairs[mask]
    return dataclasses.replace(case, cfg=dataclasses.replace(case.cfg, num_seqs=n), q=case.q[:n],
                               key=case.key[:n], value=case.value[:n], slot_mapping=case.slot_mapping[:n],
                               block_mapping=keep_pairs, block_tables=case.block_tables[:n],
                               context_lens=case.context_lens[:n])


def _oracle_caches(o, case):
    """The oracle's own copy of the pre-step caches (1-byte codes for FP8 workloads)."""
    if case.cfg.kv_dtype != "fp8_e4m3":
        return case.k_cache.clone(), case.v_cache.clone()
    nb, bs, hkv, d = case.k_cache.shape
    k8 = torch.zeros((nb, bs, hkv, d), dtype=torch.uint8)
    v8 = torch.zeros_like(k8)
    slots = torch.arange(nb * bs, dtype=torch.int64)
    o.reshape_and_cache_fp8(k8, v8, case.k_cache.view(nb * bs, hkv, d), case.v_cache.view(nb * bs, hkv, d), slots,
                            case.cfg.kv_scale, case.cfg.kv_scale)
    return k8, v8


def _oracle_step(o, case, k, v):
    if case.cfg.kv_dtype != "fp8_e4m3":
        return o.step_inplace(case, k, v)
    s = case.cfg.kv_scale
    if case.block_mapping.numel():
        o.copy_blocks(k.view(torch.bfloat16), v.view(torch.bfloat16), case.block_mapping)
    o.reshape_and_cache_fp8(k, v, case.key, case.value, case.slot_mapping, s, s)
    return o.paged_decode_fp8(case.q, k, v, s, s, case.block_tables, case.context_lens, case.scale)


def cpu_baseline(case, budget_s: float = 20.0):
    """The oracle, as it stands, on the host cores: one step on a bounded sample.
    The caches are cloned once outside the timed region (the step is idempotent)."""
    import oracle
    o = oracle.get()
    k, v = _oracle_caches(o, case)
    # calibrate on a few sequences, then size the sample to the budget
    n0 = min(4, case.cfg.num_seqs)
    t = time.perf_counter()
    _oracle_step(o, _sample_case(case, n0), k, v)
    per_seq = (time.perf_counter() - t) / n0
    n = max(1, min(case.cfg.num_seqs, int(budget_s / 2 / max(per_seq, 1e-6))))
    sample = _sample_case(case, n)
    best = None
    reps = 0
    t_all = time.perf_counter()
    while reps < 3 and (reps == 0 or time.perf_counter() - t_all < budget_s / 2):
        t = time.perf_counter()
        _oracle_step(o, sample, k, v)
        dt = time.perf_counter() - t
        best = dt if best is None else min(best, dt)
        reps += 1
    # the same step on one thread, on a sample sized to a quarter of the budget
    threads = o.num_threads
    n1 = max(1, min(n, int(budget_s / 4 / max(per_seq * threads, 1e-6))))
    sample1 = _sample_case(case, n1)
    o.set_num_threads(1)
    try:
        t = time.perf_counter()
        _oracle_step(o, sample1, k, v)
        dt1 = time.perf_counter() - t
    finally:
        o.set_num_threads(threads)
    return {"value": round(sample.kv_bytes() / best / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle", "cpu": cpu_model(), "seqs_per_s": round(n / best, 3),
            "sample": f"first {n} of {case.cfg.num_seqs} sequences of the same workload, one full step "
                      f"(copies, new-token write, fp64 decode), best of {reps}",
            "single_thread": {"value": round(sample1.kv_bytes() / dt1 / 1e9, 4), "unit": "GB/s",
                              "seqs_per_s": round(n1 / dt1, 3),
                              "sample": f"first {n1} sequences, one step, one run"}}


def run_reference(args, world, rank):
    """The fp64 oracle as the reference arm, on the host cores, rank 0 only."""
    if rank != 0:
        return None
    import oracle
    o = oracle.get()
    cfg = inputs.CONFIGS[args.workload]
    case = inputs.make_case(cfg, seed=rank_seed(cfg, 0), with_post=False)
    k, v = _oracle_caches(o, case)
    # size each step so that warm-up + timed steps take about `ref_budget` seconds
    n0 = min(4, cfg.num_seqs)
    t = time.perf_counter()
    _oracle_step(o, _sample_case(case, n0), k, v)
    per_seq = (time.perf_counter() - t) / n0
    per_step_budget = args.ref_budget / max(1, args.steps + args.warmup)
    n = max(1, min(cfg.num_seqs, int(per_step_budget / max(per_seq, 1e-6))))
    sample = _sample_case(case, n)
    for _ in range(args.warmup):
        _oracle_step(o, sample, k, v)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(o, sample, k, v)
    el = time.perf_counter() - t0
    value = sample.kv_bytes() * args.steps / el / 1e9
    desc = (f"first {n} of {cfg.num_seqs} sequences per step (copies, new-token write, fp64 decode), "
            f"{o.num_threads} threads")
    return {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(el * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "description": cfg.description, "sample_seqs_per_step": n},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": o.num_threads, "kind": "oracle", "cpu": cpu_model(),
                         "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=list(inputs.CONFIGS) + list(inputs.PREFILL_CONFIGS))
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds for the CPU-baseline sample")
    ap.add_argument("--ref-budget", type=float, default=120.0, help="seconds for the whole reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    world, rank, local = dist_setup()
    try:
        prefill = args.workload in inputs.PREFILL_CONFIGS
        if args.impl == "reference":
            line = (run_reference_prefill if prefill else run_reference)(args, world, rank)
        else:
            line = (run_prefill if prefill else run_ours)(args, world, rank, local)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
