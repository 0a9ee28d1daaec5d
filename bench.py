#!/usr/bin/env python
"""Benchmark: causal GQA attention forward TFLOP/s (bf16) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl tessera|reference]

One step = one attention forward (the whole hot path) over one batch of the
workload's synthetic inputs, already resident in HBM.  Each timed step is
preceded by an L2 flush (a 256 MB write) and timed with CUDA events on the
launching stream; the flush is outside the events.  For N > 1 (torchrun, one
rank per GPU) every rank runs the same workload on its own inputs (weak
scaling: independent batches, no collective on the data path); the reported
time is the max over ranks.

Prints one JSON line (rank 0).  ``--impl reference`` times the fp64 CPU oracle
on every host core instead, on bounded random samples of the same workload.
"""
from __future__ import annotations

import argparse
import contextlib
import dataclasses
import datetime
import itertools
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

from causal_gqa_attention_03_b200 import inputs  # noqa: E402

METRIC = "causal GQA attn fwd TFLOP/s (bf16) and % of B200 roofline vs fp64 CPU oracle"
UNIT = "TFLOP/s"
FLUSH_BYTES = 256 << 20
L2_BYTES = 126 << 20  # B200 L2
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch; rank 0 uses the workload's own seed."""
    return seed + 7919 * rank


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, period_ms: int = 100):
        self.index = index
        self.period_ms = period_ms
        self.lines = []
        self.proc = None
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=2)

    def summary(self):
        rows = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append(dict(t=t, sm=float(parts[2]), smax=float(parts[3]),
                                 power=float(parts[4]) if parts[4] not in ("[N/A]", "N/A") else None,
                                 hw=parts[6], hwt=parts[7], swt=parts[8], swp=parts[9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        inside = [r for r in rows if any(a - 0.15 <= r["t"] <= b + 0.15 for a, b in self.windows)]
        use = inside or rows
        reasons = set()
        for r in use:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in use),
                "sm_max_mhz": max(r["smax"] for r in use),
                "reasons": sorted(reasons),
                "samples": len(use),
                "samples_in_timed_region": len(inside),
                "power_w_max": max((r["power"] for r in use if r["power"] is not None), default=None)}


# --------------------------------------------------------------------- oracle
def oracle_rows_rate(w, q, k, v, seconds: float, seed: int, max_rows: int | None = None):
    """Time the fp64 oracle on random rows of the workload for about `seconds`.

    Returns (TFLOP/s, rows done, flops done, elapsed).  A row i costs
    4*d*(i+1) flops of causal attention (2*d per key for QK^T and for PV),
    summing to the metric's 2*B*Hq*T^2*d over the whole workload (up to T+1/T).
    """
    import numpy as np
    import oracle
    qb, kb, vb = inputs.bf16_bits(q), inputs.bf16_bits(k), inputs.bf16_bits(v)
    rng = np.random.default_rng(seed)
    flops = 0.0
    rows_done = 0
    t0 = time.perf_counter()
    while True:
        n = 16
        rows = np.stack([rng.integers(0, w.B, n), rng.integers(0, w.Hq, n),
                         rng.integers(0, w.T, n)], axis=1).astype(np.int64)
        rows = rows[np.lexsort((rows[:, 2], rows[:, 1], rows[:, 0]))]
        oracle.attn_rows_bf16(qb, kb, vb, rows, causal=w.causal, scale=w.scale)
        flops += float(np.sum(4.0 * w.d * (rows[:, 2] + 1)))
        rows_done += n
        el = time.perf_counter() - t0
        if el >= seconds or (max_rows is not None and rows_done >= max_rows):
            break
    return flops / el / 1e12, rows_done, flops, el


def oracle_allcore_rate(w, q, k, v, seconds: float, seed: int, threads: int | None = None,
                        run_rows: int = 128):
    """Time the fp64 oracle on every host core for about `seconds` of wall time.

    The workload's rows are cut into runs of `run_rows` consecutive rows of one
    (b, h) (oracle.fwd_runs); runs are taken in a seeded random order and
    handed to `threads` host threads (default: every core this process may
    use), each run one call of the oracle's row entry.  Submission stops once
    `seconds` have passed; the runs in flight then finish.  Returns (TFLOP/s,
    runs done, total runs, flops done, elapsed, threads); flops are the
    metric's 4*d per visible key per row (oracle.run_flops).
    """
    import numpy as np
    from concurrent.futures import ThreadPoolExecutor, FIRST_COMPLETED, wait
    import oracle
    qb, kb, vb = inputs.bf16_bits(q), inputs.bf16_bits(k), inputs.bf16_bits(v)
    threads = threads or oracle.host_threads()
    runs = oracle.fwd_runs(w.B, w.Hq, w.T, w.causal, run_rows)
    order = np.random.default_rng(seed).permutation(len(runs))

    def one(run):
        b, h, i0, i1 = run
        rows = np.empty((i1 - i0, 3), dtype=np.int64)
        rows[:, 0], rows[:, 1], rows[:, 2] = b, h, np.arange(i0, i1)
        oracle.attn_rows_bf16(qb, kb, vb, rows, causal=w.causal, scale=w.scale)
        return oracle.run_flops(run, w.d, w.T, w.causal)

    flops, done, nxt = 0.0, 0, 0
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as pool:
        pending = set()
        while nxt < len(order) and len(pending) < threads:
            pending.add(pool.submit(one, runs[order[nxt]]))
            nxt += 1
        while pending:
            fin, pending = wait(pending, return_when=FIRST_COMPLETED)
            for f in fin:
                flops += f.result()
                done += 1
            if time.perf_counter() - t0 < seconds:
                while nxt < len(order) and len(pending) < threads:
                    pending.add(pool.submit(one, runs[order[nxt]]))
                    nxt += 1
    el = time.perf_counter() - t0
    return flops / el / 1e12, done, len(runs), flops, el, threads


def config_of(w, world: int) -> dict:
    """The `config` object of the JSON line, the same in both arms."""
    return {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "causal": w.causal, "sigma_qk": w.sigma_qk, "seed": w.seed,
            "l2": "flushed before every timed step (256 MB write, outside the events)",
            "parallelism": f"dp{world} (independent batch per GPU)"}


# Host copies of small parts of the extra legs' inputs, kept for the oracle's
# timing (filled by the time_* functions).
SAMPLES = {}


def leg_cpu_baselines(w, q_h, k_h, v_h, seconds: float):
    """The fp64 oracle timed on bounded samples of each extra leg's own
    workload (single thread), in each leg's unit."""
    import numpy as np
    import oracle
    out = {}

    def timed(fn):
        n, t0 = 0, time.perf_counter()
        while True:
            fn()
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                return n, el

    # backward: random dQ rows of the headline workload (6*d*(i+1) flops each:
    # the score row, the dP row and the dQ row)
    g_h = inputs.make_grad(w.B, w.Hq, w.T, w.d, w.seed + inputs.GRAD_SEED_OFFSET)
    qb, kb, vb, gb = (inputs.bf16_bits(t) for t in (q_h, k_h, v_h, g_h))
    rng = np.random.default_rng(2)
    fl = [0.0]

    def bwd_rows():
        rows = np.stack([rng.integers(0, w.B, 8), rng.integers(0, w.Hq, 8),
                         rng.integers(0, w.T, 8)], axis=1).astype(np.int64)
        rows = rows[np.lexsort((rows[:, 2], rows[:, 1], rows[:, 0]))]
        oracle.attn_bwd_dq_rows_bf16(qb, kb, vb, gb, rows, causal=True, scale=w.scale)
        fl[0] += float(np.sum(6.0 * w.d * (rows[:, 2] + 1)))

    n, el = timed(bwd_rows)
    out["backward"] = {"value": fl[0] / el / 1e12, "unit": UNIT, "cores": 1, "kind": "oracle",
                       "sample": f"{8 * n} random dQ rows of {w.name} in {el:.1f}s "
                                 "(6*d*(i+1) flops per row), fp64, single thread"}
    for key, wd in (("decode", inputs.DECODE), ("decode_d64", inputs.DECODE_D64)):
        if key not in SAMPLES:
            continue
        qd, sk, sv, st_, sn = SAMPLES[key]
        qn, skn, svn = qd.double().numpy(), sk.double().numpy(), sv.double().numpy()
        nbytes = float(int(sn.sum()) * wd.Hkv * wd.d * 4 + 2 * len(sn) * wd.Hq * wd.d * 2)
        n, el = timed(lambda: oracle.paged_decode_f64(qn, skn, svn, st_, sn, scale=wd.scale))
        out[key] = {"value": nbytes * n / el / 1e9, "unit": "GB/s", "cores": 1,
                    "kind": "oracle",
                    "sample": f"{len(sn)} sequences ({int(sn.sum())} tokens) of {wd.name}, "
                              f"{n} steps in {el:.1f}s, fp64, single thread"}
    if "varlen" in SAMPLES:
        qv, kv, vv = (inputs.bf16_bits(t) for t in SAMPLES["varlen"])
        T = qv.shape[2]
        wv = inputs.VARLEN
        fl = [0.0]

        def vrows():
            rows = np.stack([np.zeros(8, np.int64), rng.integers(0, wv.Hq, 8),
                             rng.integers(0, T, 8)], axis=1).astype(np.int64)
            rows = rows[np.lexsort((rows[:, 2], rows[:, 1], rows[:, 0]))]
            oracle.attn_rows_bf16(qv, kv, vv, rows, causal=True, scale=wv.scale)
            fl[0] += float(np.sum(4.0 * wv.d * (rows[:, 2] + 1)))

        n, el = timed(vrows)
        out["varlen"] = {"value": fl[0] / el / 1e12, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"{8 * n} random rows of the longest sequence ({T} tokens) of "
                                   f"{wv.name} in {el:.1f}s, fp64, single thread"}
    if "prologue" in SAMPLES:
        x, wn, qkv = SAMPLES["prologue"]
        xn, wnn, qkvn = x.double().numpy(), wn.double().numpy(), qkv.double().numpy()
        n, el = timed(lambda: oracle.rmsnorm_f64(xn, wnn, 1e-6))
        rms = {"value": (4.0 * x.numel()) * n / el / 1e9, "unit": "GB/s", "cores": 1,
               "kind": "oracle", "sample": f"{x.shape[0]} rows of {x.shape[1]}, {n} times in "
                                           f"{el:.1f}s, fp64, single thread"}
        n, el = timed(lambda: oracle.rope_qkv_f64(qkvn, w.Hq, w.Hkv))
        rope = {"value": (4.0 * qkv.numel()) * n / el / 1e9, "unit": "GB/s", "cores": 1,
                "kind": "oracle", "sample": f"{qkv.shape[1]} tokens x {w.Hq + 2 * w.Hkv} heads, "
                                            f"{n} times in {el:.1f}s, fp64, single thread"}
        out["prologue"] = {"rmsnorm": rms, "rope_qkv": rope}
    return out


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    q, k, v = inputs.workload_inputs(w)
    step_seconds = 2.0
    for i in range(args.warmup):
        oracle_allcore_rate(w, q, k, v, step_seconds / 4, seed=100 + i)
    flops = 0.0
    el = 0.0
    runs = 0
    threads = 1
    for i in range(args.steps):
        _, r, total_runs, f, e, threads = oracle_allcore_rate(w, q, k, v, step_seconds,
                                                              seed=1000 + i)
        flops += f
        el += e
        runs += r
    value = flops / el / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "nproc": os.cpu_count(),
                         "sample": f"{runs} random 128-row runs of {w.name} (of {total_runs}), "
                                   f"{args.steps} steps of ~{step_seconds}s on {threads} host "
                                   "threads, fp64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------- GPU arm
def nvtx(name: str):
    """An nvtx range around one timed launch (a profiler's timeline shows
    which leg and step it belongs to); a no-op where torch lacks nvtx."""
    import torch
    try:
        return torch.cuda.nvtx.range(name)
    except (AttributeError, RuntimeError):
        return contextlib.nullcontext()


def time_kernel(w, q, k, v, steps, warmup, flush, stream, tess, torch):
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device=q.device)
    launches = 0
    for _ in range(warmup):
        flush.zero_()
        tess.attn_fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        starts[i].record(stream)
        with nvtx(f"attn_fwd {w.name} step {i}"):
            tess.attn_fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse,
                          stream=stream)
        launches += tess.tessera_attn_last_launch_count()
        ends[i].record(stream)
    torch.cuda.synchronize()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    return times, launches, o, lse


def time_back_to_back(w, q, k, v, n, stream, tess, torch):
    """Mean time of n forward launches queued back to back (no L2 flush
    between them: the warm-L2 figure, and for tiny workloads the launch
    rate), one CUDA-event pair around all of them."""
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device=q.device)
    for _ in range(3):
        tess.attn_fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        tess.attn_fwd(q, k, v, causal=w.causal, scale=w.scale, out=o, lse=lse, stream=stream)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def time_empty_launches(n, stream, torch):
    """Mean time of n empty kernels (torch's 0-cycle sleep) queued back to
    back on `stream`: the launch floor of the device and driver."""
    with torch.cuda.stream(stream):
        for _ in range(10):
            torch.cuda._sleep(0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(n):
            torch.cuda._sleep(0)
        b.record(stream)
        torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def time_backward(w, q, k, v, g, steps, warmup, flush, stream, tess, torch):
    """The backward (3 launches: D prep, dK/dV, dQ) on the forward's O and
    LSE, each step after an L2 flush, CUDA events around the three
    launches."""
    o, lse = tess.attn_fwd(q, k, v, causal=w.causal, scale=w.scale, stream=stream)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    nbytes = tess.tessera_attn_bwd_workspace_bytes_kv(w.B, w.Hq, w.Hkv, w.T, w.d)
    ws = torch.empty((nbytes + 3) // 4, dtype=torch.float32, device=q.device)

    def call():
        tess.attn_bwd(q, k, v, o, lse, g, causal=w.causal, scale=w.scale, dq=dq, dk=dk, dv=dv,
                      workspace=ws, stream=stream)

    for _ in range(warmup):
        flush.zero_()
        call()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    launches = 0
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        starts[i].record(stream)
        with nvtx(f"{call.__qualname__.split('.')[0]} step {i}"):
            call()
        launches += tess.tessera_attn_last_launch_count()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [s_.elapsed_time(e) for s_, e in zip(starts, ends)], launches, nbytes


def time_decode(wd, steps, warmup, flush, stream, tess, torch, dev, sample_key="decode"):
    """One decode step over the paged cache of ``wd`` (2 launches: the split-KV
    partial kernel and the merge), CUDA events around both launches.  The
    step reads far more than L2 holds (2.43 GB for the serving batch), so
    the timed steps run back to back with no flush; a 256 MB write flush
    before each step would add the write-back of its dirty lines to the
    step.  A second, shorter series with that flush is timed for reference.
    Returns (per-step ms list, launches, workspace bytes, per-step ms list
    with the write flush)."""
    q, kc, vc, table, lens = inputs.make_paged_device(wd, dev)
    o = torch.empty_like(q)
    lse = torch.empty((wd.B, wd.Hq), dtype=torch.float32, device=dev)
    nbytes = tess.tessera_attn_decode_workspace_bytes(wd.B, wd.Hq, wd.max_len, wd.d)
    ws = torch.empty((nbytes + 3) // 4, dtype=torch.float32, device=dev)

    def call():
        tess.attn_decode(q, kc, vc, table, lens, max_seq_len=wd.max_len, scale=wd.scale, out=o,
                         lse=lse, workspace=ws, stream=stream)

    for _ in range(warmup):
        call()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    launches = 0
    torch.cuda.synchronize()
    for i in range(steps):
        starts[i].record(stream)
        with nvtx(f"{call.__qualname__.split('.')[0]} step {i}"):
            call()
        launches += tess.tessera_attn_last_launch_count()
        ends[i].record(stream)
    torch.cuda.synchronize()
    nf = min(steps, 20)
    fs = [torch.cuda.Event(enable_timing=True) for _ in range(nf)]
    fe = [torch.cuda.Event(enable_timing=True) for _ in range(nf)]
    for i in range(nf):
        flush.zero_()
        fs[i].record(stream)
        call()
        fe[i].record(stream)
    torch.cuda.synchronize()
    # two sequences of the batch, copied to the host, for the oracle's timing
    tab_h, lens_h = table.cpu().numpy(), lens.cpu().numpy()
    pick = [int(lens_h.argmax()), int(len(lens_h) // 2)]
    sk, sv, st_, sn = inputs.gather_sequences(tab_h, lens_h, pick, wd.bs, kc, vc)
    SAMPLES[sample_key] = (q[pick].cpu(), sk, sv, st_, sn)
    del q, kc, vc, table, lens, o, lse, ws
    return ([s_.elapsed_time(e) for s_, e in zip(starts, ends)], launches, nbytes,
            [s_.elapsed_time(e) for s_, e in zip(fs, fe)])


def time_prologue(w, steps, warmup, flush, stream, tess, torch, dev):
    """RMSNorm of the hidden states [B*T, Hq*d] and the rotary embedding with
    head split of the projection output [B, T, (Hq + 2 Hkv) d], at the
    workload's sizes, each timed alone (one launch per step, L2 flushed
    before each).  Returns {name: (per-step ms list, bytes per step)}."""
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 17)
    dm = w.Hq * w.d
    rows = w.B * w.T
    x = torch.randn((rows, dm), generator=g, device=dev).to(torch.bfloat16)
    wn = torch.randn((dm,), generator=g, device=dev).to(torch.bfloat16)
    y = torch.empty_like(x)
    h3 = w.Hq + 2 * w.Hkv
    qkv = torch.randn((w.B, w.T, h3 * w.d), generator=g, device=dev).to(torch.bfloat16)
    q = torch.empty((w.B, w.Hq, w.T, w.d), dtype=torch.bfloat16, device=dev)
    k = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    legs = {
        "rmsnorm": (lambda: tess.rmsnorm(x, wn, 1e-6, out=y, stream=stream),
                    2 * rows * dm * 2 + dm * 2),
        "rope_qkv": (lambda: tess.rope_qkv(qkv, w.Hq, w.Hkv, q=q, k=k, v=v, stream=stream),
                     2 * w.B * w.T * h3 * w.d * 2),
    }
    out = {}
    for name, (call, nbytes) in legs.items():
        for _ in range(warmup):
            flush.zero_()
            call()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        torch.cuda.synchronize()
        launches = 0
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            call()
            launches += tess.tessera_attn_last_launch_count()
            ends[i].record(stream)
        torch.cuda.synchronize()
        out[name] = ([s_.elapsed_time(e) for s_, e in zip(starts, ends)], nbytes, launches)
    SAMPLES["prologue"] = (x[:64].cpu(), wn.cpu(), qkv[:, :16].contiguous().cpu())
    del x, wn, y, qkv, q, k, v
    return out


def prologue_line(w, res, peaks, peak_src):
    hbm = float(peaks["hbm_gbs"])
    line = {"metric": "attention prologue GB/s (bf16): RMSNorm, RoPE + head split",
            "config": {"rows": w.B * w.T, "hidden": w.Hq * w.d, "B": w.B, "T": w.T, "Hq": w.Hq,
                       "Hkv": w.Hkv, "d": w.d, "eps": 1e-6, "rope_base": 10000.0,
                       "positions": "t (none given)"},
            "l2": "flushed before every timed step"}
    for name, (times, nbytes, launches) in res.items():
        ms = statistics.median(times)
        gbs = nbytes / (ms * 1e-3) / 1e9
        line[name] = {"value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 5),
                      "bytes_per_step": nbytes, "gpu_launches": launches,
                      "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm,
                                   "unit": "GB/s", "frac": round(gbs / hbm, 4),
                                   "traffic": traffic_bytes(name, w.name),
                                   "peak_source": f"{peak_src} hbm_gbs"}}
    return line


def time_varlen(wv, steps, warmup, flush, stream, tess, torch, dev):
    """The packed variable-length forward over ``wv``'s mixed lengths, drawn
    on the device (CUDA generator seeded with the workload's seed), one
    launch per step, L2 flushed before each."""
    lens = wv.lens()
    total = sum(lens)
    g = torch.Generator(device=dev)
    g.manual_seed(wv.seed)
    q = torch.randn((total, wv.Hq, wv.d), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((total, wv.Hkv, wv.d), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((total, wv.Hkv, wv.d), generator=g, device=dev).to(torch.bfloat16)
    cu = torch.tensor([0] + list(itertools.accumulate(lens)), dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((wv.Hq, total), dtype=torch.float32, device=dev)

    def call():
        tess.attn_fwd_varlen(q, k, v, cu, max(lens), causal=True, scale=wv.scale, out=o,
                             lse=lse, stream=stream)

    for _ in range(warmup):
        flush.zero_()
        call()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    launches = 0
    torch.cuda.synchronize()
    for i in range(steps):
        flush.zero_()
        starts[i].record(stream)
        with nvtx(f"{call.__qualname__.split('.')[0]} step {i}"):
            call()
        launches += tess.tessera_attn_last_launch_count()
        ends[i].record(stream)
    torch.cuda.synchronize()
    b = max(range(len(lens)), key=lambda i: lens[i])
    s0 = sum(lens[:b])
    SAMPLES["varlen"] = tuple(t[s0:s0 + lens[b]].permute(1, 0, 2).contiguous()[None].cpu()
                              for t in (q, k, v))
    del q, k, v, o, lse
    return [s_.elapsed_time(e) for s_, e in zip(starts, ends)], launches


def noncausal_line(wn, times, max_ms, steps, launches, world, peaks, peak_src):
    """The full-attention (causal = 0) forward on the headline workload's
    inputs: TFLOP/s of 4*B*Hq*T^2*d against the measured bf16 peak."""
    value = wn.flops * steps * world / (max_ms * 1e-3) / 1e12
    achieved = wn.flops / (statistics.mean(times) * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    return {"metric": "GQA attn fwd TFLOP/s (bf16), full attention (no causal mask)",
            "value": round(value, 2), "unit": UNIT, "steps": steps,
            "ms_per_step": round(max_ms / steps, 5), "flops_per_step": wn.flops,
            "flop_count": "4*B*Hq*T^2*d: QK^T and PV over every key",
            "config": {"workload": wn.name, "B": wn.B, "T": wn.T, "Hq": wn.Hq, "Hkv": wn.Hkv,
                       "d": wn.d, "causal": False},
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                         "unit": UNIT, "frac": round(achieved / peak, 4),
                         "traffic": traffic_bytes("noncausal", wn.name),
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         **nominal_roofline(achieved, wn)},
            "gpu_launches": launches, "l2": "flushed before every timed step"}


def varlen_line(wv, times, launches, peaks, peak_src):
    ms = statistics.median(times)
    tf = wv.flops / (ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    return {"metric": "packed variable-length causal GQA attn fwd TFLOP/s (bf16)",
            "value": round(tf, 2), "unit": UNIT, "ms": round(ms, 5), "steps": len(times),
            "flops_per_step": wv.flops,
            "flop_count": "sum over sequences of the metric's 2*Hq*T_b^2*d",
            "config": wv.describe(), "gpu_launches": launches,
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peak,
                         "unit": UNIT, "frac": round(tf / peak, 4), "traffic": traffic_bytes("varlen", wv.name),
                         "peak_source": f"{peak_src} bf16_tflops (burst)"},
            "l2": "flushed before every timed step"}


def time_e2e(w, q_h, k_h, v_h, steps, warmup, stream, tess, torch, dev):
    """Public API end to end: pinned host Q/K/V in, pinned host O/LSE out, through
    tessera_attn_fwd_host (copies pipelined with the kernels over pieces of
    query heads, the library's default plan).  Each step returns with the outputs on the host."""
    staging = {"q": torch.empty(q_h.shape, dtype=torch.bfloat16, device=dev),
               "k": torch.empty(k_h.shape, dtype=torch.bfloat16, device=dev),
               "v": torch.empty(k_h.shape, dtype=torch.bfloat16, device=dev),
               "o": torch.empty(q_h.shape, dtype=torch.bfloat16, device=dev),
               "lse": torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, device=dev)}
    o_h = torch.empty(q_h.shape, dtype=torch.bfloat16, pin_memory=True)
    l_h = torch.empty((w.B, w.Hq, w.T), dtype=torch.float32, pin_memory=True)

    def step():
        tess.attn_fwd_host(q_h, k_h, v_h, causal=w.causal, scale=w.scale, out=o_h, lse=l_h,
                           staging=staging, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        with nvtx(f"attn_fwd_host {w.name} step {i}"):
            step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    h2d = (q_h.numel() + k_h.numel() + v_h.numel()) * 2
    d2h = o_h.numel() * 2 + l_h.numel() * 4
    return ms, h2d, d2h


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=inputs.LARGEST, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="tessera", choices=["tessera", "reference"])
    ap.add_argument("--no-sweep", action="store_true", help="skip the per-workload sweep")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--only", choices=["forward", "backward", "decode", "decode_d64", "noncausal",
                                       "prologue", "varlen"],
                    help="time one extra leg alone and print its object (for profiling it)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = inputs.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    import causal_gqa_attention_03_b200 as tess

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=datetime.timedelta(seconds=120))
    tess.load_library()
    if args.only:
        return one_leg(args, tess, torch, dev, world, rank, local)

    q_h, k_h, v_h = inputs.make_qkv(w.B, w.Hq, w.Hkv, w.T, w.d,
                                    rank_seed(w.seed, rank), w.sigma_qk)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    times, launches, _, _ = time_kernel(w, q, k, v, args.steps, args.warmup, flush, stream,
                                        tess, torch)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    clocks.mark(t_wall0, t_wall1)
    err = tess.tessera_attn_device_error()
    if err != 0:
        raise SystemExit(f"device-side wait gave up (code {err})")

    kernel_ms = sum(times)
    max_ms = max_over_ranks(kernel_ms, dev)
    total_flops = w.flops * args.steps * world
    value = total_flops / (max_ms * 1e-3) / 1e12
    ms_per_step = max_ms / args.steps
    per_launch_ms = statistics.mean(times)
    achieved = w.flops / (per_launch_ms * 1e-3) / 1e12

    # end to end through the public API with pinned host buffers
    q_pin, k_pin, v_pin = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    e2e_ms, h2d, d2h = time_e2e(w, q_pin, k_pin, v_pin, args.e2e_steps, 3, stream, tess, torch,
                                dev)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    e2e_value = w.flops * world / (e2e_ms * 1e-3) / 1e12

    # the backward on the same inputs (dO drawn from its own seeded generator)
    g = inputs.make_grad(w.B, w.Hq, w.T, w.d,
                         rank_seed(w.seed, rank) + inputs.GRAD_SEED_OFFSET).to(dev)
    bwd_steps = max(5, min(args.steps, int(0.5 / max(2.5 * w.flops / 5e14, 1e-6))))
    bwd_times, bwd_launches, bwd_ws = time_backward(w, q, k, v, g, bwd_steps, 3, flush, stream,
                                                    tess, torch)
    bwd_max_ms = max_over_ranks(sum(bwd_times), dev)
    err = tess.tessera_attn_device_error()
    if err != 0:
        raise SystemExit(f"device-side wait gave up in the backward (code {err})")

    # one decode step over a paged K/V cache (its own synthetic serving batch)
    wd = inputs.DECODE
    dec_steps = max(5, min(args.steps, 200))
    dec_times, dec_launches, dec_ws, dec_flushed = time_decode(wd, dec_steps, 3, flush, stream,
                                                               tess, torch,
                                                  dev)
    dec_max_ms = max_over_ranks(sum(dec_times), dev)
    err = tess.tessera_attn_device_error()
    if err != 0:
        raise SystemExit(f"device-side error in the decode step (code {err})")

    # the same serving batch at head dimension 64
    wd64 = inputs.DECODE_D64
    d64_times, d64_launches, d64_ws, d64_flushed = time_decode(
        wd64, dec_steps, 3, flush, stream, tess, torch, dev, sample_key="decode_d64")
    d64_max_ms = max_over_ranks(sum(d64_times), dev)
    err = tess.tessera_attn_device_error()
    if err != 0:
        raise SystemExit(f"device-side error in the d=64 decode step (code {err})")

    # the headline workload without the causal mask (full attention)
    wn = dataclasses.replace(w, causal=False, name=w.name + "_noncausal")
    nc_steps = max(5, min(args.steps, 50))
    nc_times, nc_launches, _, _ = time_kernel(wn, q, k, v, nc_steps, 3, flush, stream, tess,
                                              torch)
    nc_max_ms = max_over_ranks(sum(nc_times), dev)

    # the packed variable-length forward on its mixed-length batch
    vl_times, vl_launches = time_varlen(inputs.VARLEN, max(5, min(args.steps, 50)), 3, flush,
                                        stream, tess, torch, dev)

    # the prologue kernels at the workload's sizes
    pro = time_prologue(w, max(5, min(args.steps, 100)), 3, flush, stream, tess, torch, dev)

    sweep = {}
    if not args.no_sweep and world == 1:
        for name, ws in inputs.WORKLOADS.items():
            qs, ks, vs = (t.to(dev) for t in inputs.workload_inputs(ws))
            if name == w.name:
                sweep[name] = {"tflops": round(value, 1), "ms": round(ms_per_step, 4)}
            else:
                n = max(5, min(200, int(0.5 / max(ws.flops / 1.2e15, 1e-6))))
                ts, _, _, _ = time_kernel(ws, qs, ks, vs, n, 3, flush, stream, tess, torch)
                ms = statistics.median(ts)
                sweep[name] = {"tflops": round(ws.flops / (ms * 1e-3) / 1e12, 1),
                               "ms": round(ms, 4)}
            # warm L2 (no flush between launches); 1000 launches for the
            # launch-bound smallest workloads
            nb = 1000 if ws.flops < 1e9 else max(5, min(200, int(0.3 / max(ws.flops / 1.2e15, 1e-6))))
            warm = time_back_to_back(ws, qs, ks, vs, nb, stream, tess, torch)
            sweep[name]["warm_ms"] = round(warm, 4)
            sweep[name]["warm_tflops"] = round(ws.flops / (warm * 1e-3) / 1e12, 1)
            sweep[name]["warm_launches"] = nb
            if ws.flops < 1e9:
                # the launch floor on the same stream: an empty kernel (torch's
                # 0-cycle sleep) back to back, for the tiny workload's context
                sweep[name]["empty_launch_ms"] = round(time_empty_launches(1000, stream, torch), 4)
            gs = inputs.workload_grad(ws).to(dev)
            n = max(5, min(100, int(0.3 / max(2.5 * ws.flops / 5e14, 1e-6))))
            tb, _, _ = time_backward(ws, qs, ks, vs, gs, n, 3, flush, stream, tess, torch)
            mb = statistics.median(tb)
            sweep[name]["bwd_tflops"] = round(2.5 * ws.flops / (mb * 1e-3) / 1e12, 1)
            sweep[name]["bwd_ms"] = round(mb, 4)
            del qs, ks, vs, gs
        err = tess.tessera_attn_device_error()
        if err != 0:
            raise SystemExit(f"device-side wait gave up in the sweep (code {err})")

    clocks.stop()
    clk = clocks.summary()

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    traffic = traffic_bytes("forward", w.name)
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                "unit": UNIT, "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": f"{peak_src} bf16_tflops (burst, kernel timed alone)",
                "flops_per_launch": w.flops, "io_bytes_per_launch": w.io_bytes,
                **nominal_roofline(achieved, w)}
    if "bf16_tflops_sustained" in peaks:
        # long runs settle at the power cap: the sustained GEMM figure beside it
        roofline["frac_of_sustained"] = round(achieved / float(peaks["bf16_tflops_sustained"]), 4)

    cpu = None
    leg_cpu = {}
    if not args.no_cpu_baseline and world == 1:
        rate, runs, total_runs, fl, el, threads = oracle_allcore_rate(
            w, q_h, k_h, v_h, args.cpu_seconds, seed=1)
        rate1, rows1, _, el1 = oracle_rows_rate(w, q_h, k_h, v_h, 3.0, seed=1)
        cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
               "nproc": os.cpu_count(),
               "sample": f"{runs} random 128-row runs of {w.name} ({100.0 * fl / w.flops:.1f}% "
                         f"of its flops, {runs} of {total_runs} runs) in {el:.1f}s on "
                         f"{threads} host threads, fp64",
               "single_thread": {"value": rate1, "unit": UNIT, "cores": 1,
                                 "sample": f"{rows1} random (b,h,i) rows in {el1:.1f}s"}}
        leg_cpu = leg_cpu_baselines(w, q_h, k_h, v_h, seconds=3.0)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(w, world),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "path": "tessera_attn_fwd_host: pinned host Q/K/V -> per piece of query heads "
                        "(default plan: 8 even pieces, the last cut down to one-head pieces; "
                        "H2D copy, kernel on one of four streams, D2H copy; copies overlap "
                        "kernels) -> pinned host O/LSE",
                "pieces": len(tess.tessera_attn_fwd_host_plan(w.B, w.Hq, w.Hkv, 0))},
        "gpu_launches": launches,
        "backward": backward_line(w, bwd_times, bwd_max_ms, bwd_steps, bwd_launches, bwd_ws,
                                  world, peaks, peak_src),
        "decode": decode_line(wd, dec_times, dec_max_ms, dec_steps, dec_launches, dec_ws, world,
                              peaks, peak_src, dec_flushed),
        "decode_d64": decode_line(wd64, d64_times, d64_max_ms, dec_steps, d64_launches, d64_ws,
                                  world, peaks, peak_src, d64_flushed),
        "noncausal": noncausal_line(wn, nc_times, nc_max_ms, nc_steps, nc_launches, world,
                                    peaks, peak_src),
        "varlen": varlen_line(inputs.VARLEN, vl_times, vl_launches, peaks, peak_src),
        "prologue": prologue_line(w, pro, peaks, peak_src),
        "clocks": clk,
        "sweep": sweep or None,
    }
    for leg, base in leg_cpu.items():
        if leg == "prologue":
            for kname, kb_ in base.items():
                line["prologue"][kname]["cpu_baseline"] = kb_
        else:
            line[leg]["cpu_baseline"] = base
    print(json.dumps(line), flush=True)
    return 0


def one_leg(args, tess, torch, dev, world, rank, local):
    """--only LEG: one of the extra legs alone, one JSON line with its object."""
    import torch.distributed as dist
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t0 = time.time()
    w = inputs.WORKLOADS[args.workload]
    if args.only == "forward":
        q, k, v = (t.to(dev) for t in inputs.make_qkv(w.B, w.Hq, w.Hkv, w.T, w.d,
                                                     rank_seed(w.seed, rank), w.sigma_qk))
        times, launches, _, _ = time_kernel(w, q, k, v, args.steps, args.warmup, flush, stream,
                                            tess, torch)
        max_ms = max_over_ranks(sum(times), dev)
    elif args.only == "backward":
        q, k, v = (t.to(dev) for t in inputs.make_qkv(w.B, w.Hq, w.Hkv, w.T, w.d,
                                                     rank_seed(w.seed, rank), w.sigma_qk))
        g = inputs.make_grad(w.B, w.Hq, w.T, w.d,
                             rank_seed(w.seed, rank) + inputs.GRAD_SEED_OFFSET).to(dev)
        times, launches, ws = time_backward(w, q, k, v, g, args.steps, args.warmup, flush,
                                            stream, tess, torch)
        max_ms = max_over_ranks(sum(times), dev)
    elif args.only in ("decode", "decode_d64"):
        wd = inputs.DECODE if args.only == "decode" else inputs.DECODE_D64
        times, launches, ws, flushed = time_decode(wd, args.steps, args.warmup, flush, stream,
                                                   tess, torch, dev)
        max_ms = max_over_ranks(sum(times), dev)
    elif args.only == "noncausal":
        wn = dataclasses.replace(w, causal=False, name=w.name + "_noncausal")
        q, k, v = (t.to(dev) for t in inputs.make_qkv(w.B, w.Hq, w.Hkv, w.T, w.d,
                                                     rank_seed(w.seed, rank), w.sigma_qk))
        times, launches, _, _ = time_kernel(wn, q, k, v, args.steps, args.warmup, flush, stream,
                                            tess, torch)
        max_ms = max_over_ranks(sum(times), dev)
    elif args.only == "varlen":
        times, launches = time_varlen(inputs.VARLEN, args.steps, args.warmup, flush, stream, tess,
                                      torch, dev)
    else:
        pro = time_prologue(inputs.WORKLOADS[args.workload], args.steps, args.warmup, flush,
                            stream, tess, torch, dev)
    t1 = time.time()
    clocks.mark(t0, t1)
    err = tess.tessera_attn_device_error()
    if err != 0:
        raise SystemExit(f"device-side error in the {args.only} leg (code {err})")
    clocks.stop()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peaks, peak_src = load_peaks()
    if args.only == "forward":
        achieved = w.flops / (statistics.mean(times) * 1e-3) / 1e12
        peak = float(peaks["bf16_tflops"])
        line = {"metric": METRIC, "value": round(w.flops * args.steps * world / (max_ms * 1e-3) / 1e12, 2),
                "unit": UNIT, "steps": args.steps, "ms_per_step": round(max_ms / args.steps, 5),
                "config": config_of(w, world), "gpu_launches": launches,
                "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                             "unit": UNIT, "frac": round(achieved / peak, 4), "traffic": traffic_bytes("forward", w.name),
                             "peak_source": f"{peak_src} bf16_tflops (burst)",
                             **nominal_roofline(achieved, w)}}
    elif args.only == "backward":
        line = backward_line(w, times, max_ms, args.steps, launches, ws, world, peaks, peak_src)
        line["config"] = {"workload": args.workload}
    elif args.only in ("decode", "decode_d64"):
        line = decode_line(wd, times, max_ms, args.steps, launches, ws, world, peaks, peak_src,
                           flushed)
    elif args.only == "noncausal":
        line = noncausal_line(wn, times, max_ms, args.steps, launches, world, peaks, peak_src)
    elif args.only == "varlen":
        line = varlen_line(inputs.VARLEN, times, launches, peaks, peak_src)
    else:
        line = prologue_line(inputs.WORKLOADS[args.workload], pro, peaks, peak_src)
    line.update({"n_gpus": world, "warmup": args.warmup, "higher_is_better": True,
                 "scaling": "weak", "dtype": "bf16", "data": "synthetic",
                 "clocks": clocks.summary()})
    print(json.dumps(line), flush=True)
    return 0


def backward_line(w, times, max_ms, steps, launches, ws_bytes, world, peaks, peak_src):
    """The backward's object of the JSON line: tensor-bound, TFLOP/s of the
    five products over the causal triangle against the measured bf16 peak.
    The kernels issue seven (the dQ kernel recomputes S and dP)."""
    flops = 2.5 * w.flops
    value = flops * steps * world / (max_ms * 1e-3) / 1e12
    achieved = flops / (statistics.mean(times) * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    return {"metric": "causal GQA attn bwd TFLOP/s (bf16)", "value": round(value, 2),
            "unit": UNIT, "steps": steps, "ms_per_step": round(max_ms / steps, 5),
            "flops_per_step": flops,
            "flop_count": "5*B*Hq*T^2*d: five products over the causal triangle, "
                          "counted as the forward's 2*B*Hq*T^2*d counts two",
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                         "unit": UNIT, "frac": round(achieved / peak, 4), "traffic": traffic_bytes("backward", w.name),
                         "peak_source": f"{peak_src} bf16_tflops (burst)",
                         "issued_flops_per_step": 3.5 * w.flops,
                         "issued_frac": round(1.4 * achieved / peak, 4)},
            "gpu_launches": launches, "workspace_bytes": ws_bytes,
            "l2": "flushed before every timed step"}


def decode_line(wd, times, max_ms, steps, launches, ws_bytes, world, peaks, peak_src,
                flushed=None):
    """The decode step's object of the JSON line: HBM-bound, so GB/s of the
    bytes a step must move (io_bytes) against the measured copy bandwidth."""
    nbytes = wd.io_bytes()
    value = nbytes * steps * world / (max_ms * 1e-3) / 1e9
    per_step = statistics.mean(times)
    achieved = nbytes / (per_step * 1e-3) / 1e9
    hbm = float(peaks["hbm_gbs"])
    return {"metric": "paged-KV GQA decode step GB/s (bf16 cache)", "value": round(value, 1),
            "unit": "GB/s", "steps": steps, "ms_per_step": round(max_ms / steps, 5),
            "config": wd.describe(),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": traffic_bytes("decode" if wd.d == 128 else "decode_d64", wd.name),
                         "peak_source": f"{peak_src} hbm_gbs",
                         "bytes_per_step": nbytes,
                         "byte_count": "K and V rows of every cached token, q, o, lse, "
                                       "lengths and the block ids read"},
            "gpu_launches": launches, "workspace_bytes": ws_bytes,
            "l2": f"no flush: the step reads {nbytes / 1e9:.2f} GB, "
                  f"{nbytes / L2_BYTES:.0f}x what L2 holds; the peak is a copy (read + write) "
                  "rate and the step mostly reads",
            "ms_per_step_write_flush": (round(statistics.median(flushed), 5) if flushed else None),
            "write_flush_note": "a 256 MB write before each step, outside the events: its dirty "
                                "lines are written back during the step"}


def nominal_roofline(achieved: float, w) -> dict:
    """The target's own roofline for a forward launch: the lesser of the
    nominal dense bf16 rate (2.25 PFLOP/s) and the I/O bytes (Q, K, V, O, LSE)
    over a nominal 8 TB/s, with the target of 60 % of it for the largest
    causal workload."""
    roof = min(NOMINAL_BF16_TFLOPS, w.flops / w.io_bytes * NOMINAL_HBM_GBS * 1e9 / 1e12)
    frac = achieved / roof
    return {"nominal_peak": round(roof, 1), "frac_nominal": round(frac, 4),
            "target_frac_nominal": 0.60, "target_met": bool(frac >= 0.60)}


# The kernel headers each leg is built from: a leg's DRAM-traffic record in
# profiles/traffic.json stays valid while they are unchanged.
_FWD_SOURCES = ["attn_fwd_sm100.cuh", "exp2_fma.cuh", "sm100_ptx.cuh"]
LEG_SOURCES = {"forward": _FWD_SOURCES, "varlen": _FWD_SOURCES, "noncausal": _FWD_SOURCES,
               "backward": ["attn_bwd_sm100.cuh"] + _FWD_SOURCES,
               "decode": ["paged_decode_tc.cuh", "paged_decode.cuh"] + _FWD_SOURCES,
               "decode_d64": ["paged_decode_tc.cuh", "paged_decode.cuh"] + _FWD_SOURCES,
               "rmsnorm": ["prologue.cuh"], "rope_qkv": ["prologue.cuh"]}


def kernel_source_sha(leg: str = "forward") -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "causal_gqa_attention_03_b200", "csrc")
    for name in LEG_SOURCES[leg]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_bytes(leg: str, workload: str):
    """DRAM bytes (read + write) per launch of the leg's kernels, from the
    one-pass ncu capture recorded in profiles/traffic.json; None when there is
    no record for this workload or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get("records", {}).get(leg)
    if (not rec or not str(rec.get("workload", "")).startswith(workload)
            or rec.get("kernel_source_sha") != kernel_source_sha(leg)):
        return None
    return rec.get("bytes_per_launch")


if __name__ == "__main__":
    sys.exit(main())
