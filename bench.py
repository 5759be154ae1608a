"""Benchmark of the paged-attention decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the new tokens' cache write
(pa_reshape_and_cache; plus pa_copy_blocks for the shared-prefix workload) followed by the
decode (pa_decode).  The default workload is the Llama-3-8B-shaped decode step: 64 sequences,
32 query / 8 KV heads, head_dim 128, bf16, block_size 16, contexts U[128, 2048].

`value` is the whole-job throughput in algorithmic GB/s: the bytes a step must move (every
attended K/V row once, Q and out, block-table entries, context lengths, the written rows), with
inputs resident in HBM.  To keep L2 (126 MB) from serving repeated reads, consecutive steps
rotate over several copies of the KV pool whose attended bytes each exceed L2.  `e2e` is the
same metric measured through the same public calls with the step's inputs copied from pinned
host memory and the output read back every step.  `roofline` relates the decode kernel's
algorithmic bytes per launch to its mean CUDA-event duration and the measured HBM copy
bandwidth.  `cpu_baseline` times the CPU oracle on a bounded sample of the same workload.

With --gpus N (launched under torchrun) every rank runs an independent replica of the step on
its own GPU: the path has no exchange step, so there is no collective on the data path.
--impl reference times the CPU oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_427_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention KV GB/s (% of B200 HBM peak), attended tokens/s"
PREFILL_METRIC = "paged prefill attention TFLOP/s, new tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20
ELT = {"f32": 4, "bf16": 2, "f16": 2}


# ----------------------------------------------------------------------------------------------
# byte accounting
# ----------------------------------------------------------------------------------------------

def decode_bytes(b: W.PagedBatch, out_elt: int, unique: bool = True, kv_elt: int | None = None) -> int:
    """Algorithmic bytes of one decode: each attended K/V row once (a physical slot shared by
    several sequences counts once when `unique`), Q and out rows, the block-table entries of
    each context and the context lengths.  kv_elt: bytes per cache element when the cache is
    stored in another type than the batch's (FP8: 1), plus the per-head scales."""
    e = ELT[b.dtype]
    ekv = e if kv_elt is None else kv_elt
    lens = np.maximum(b.context_lens.astype(np.int64), 0)
    row = b.num_kv_heads * b.head_dim * ekv * 2  # K and V of one token, all kv heads
    if unique:
        slots = []
        for s, L in enumerate(lens):
            if L:
                t = np.arange(L)
                slots.append(b.block_tables[s, t // b.block_size].astype(np.int64) * b.block_size
                             + t % b.block_size)
        kv = (len(np.unique(np.concatenate(slots))) if slots else 0) * row
    else:
        kv = int(lens.sum()) * row
    qo = b.num_seqs * b.num_heads * b.head_dim * (e + out_elt)
    tables = int(((lens + b.block_size - 1) // b.block_size).sum()) * 4 + b.num_seqs * 4
    scales = 0 if kv_elt is None else b.num_kv_heads * 4 * 2
    return int(kv + qo + tables + scales)


def write_bytes(b: W.PagedBatch) -> int:
    """New K/V rows read and stored, their slots, and whole-block copies (read + write)."""
    e = ELT[b.dtype]
    t = int((b.slot_mapping >= 0).sum())
    rows = t * b.num_kv_heads * b.head_dim * e * 2 * 2 + len(b.slot_mapping) * 8
    copies = 0
    if b.block_mapping is not None:
        copies = len(b.block_mapping) * (b.num_kv_heads * b.block_size * b.head_dim * e * 2 * 2 + 16)
    return int(rows + copies)


def attended_bytes(b: W.PagedBatch) -> int:
    lens = np.maximum(b.context_lens.astype(np.int64), 0)
    return int(lens.sum()) * b.num_kv_heads * b.head_dim * ELT[b.dtype] * 2


# ----------------------------------------------------------------------------------------------
# environment facts
# ----------------------------------------------------------------------------------------------

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCES = ("pa_decode_mma.cuh", "pa_decode_common.cuh", "pa_decode.cuh", "pa_device.cuh",
                  "pa_internal.h", "pa_decode_bf16_d128.cu")


def kernel_sources_digest() -> str:
    """Digest of the files the 16-bit decode kernels are compiled from (device code and the
    argument block), not the host-side API or the other kernels."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_427_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f in DECODE_SOURCES:
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken on the
    current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        entry = rec.get(workload)
        if entry and entry.get("sources") == kernel_sources_digest():
            return float(entry["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the GPU works."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.gpu_id = gpu_id

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
                power.append(float(p[3]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        # samples under load: the upper half by power draw
        cut = statistics.median(power)
        loaded = [s for s, pw in zip(sm, power) if pw >= cut] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power)}


# ----------------------------------------------------------------------------------------------
# the oracle (CPU baseline and reference arm)
# ----------------------------------------------------------------------------------------------

def oracle_sample_run(b: W.PagedBatch, budget_s: float, orc, num_threads: int = 0):
    """Time the oracle's step on the first n sequences, n grown until one run takes about
    budget_s (num_threads 0: all the oracle's OpenMP threads).  Returns (seconds, n,
    algorithmic bytes of the sample, attended tokens)."""
    kc, vc = b.key_cache, b.value_cache
    n = 1
    while True:
        sub = W.sub_batch(b, np.arange(n))
        t0 = time.perf_counter()
        orc.decode(sub["query"], kc, vc, sub["block_tables"], sub["context_lens"], b.scale, b.dtype,
                   num_threads=num_threads)
        dt = time.perf_counter() - t0
        if dt >= budget_s or n == b.num_seqs:
            break
        n = min(b.num_seqs, max(n + 1, int(n * min(8.0, budget_s / max(dt, 1e-4)))))
    sb = W.PagedBatch(**{**b.__dict__, "query": sub["query"], "block_tables": sub["block_tables"],
                          "context_lens": sub["context_lens"]})
    return dt, n, decode_bytes(sb, ELT[b.dtype], unique=False), int(sub["context_lens"].sum())


def cpu_baseline(b: W.PagedBatch, budget_s: float = 10.0):
    import oracle

    orc = oracle.load()
    dt, n, nbytes, toks = oracle_sample_run(b, budget_s, orc)
    # the same oracle on one thread, over a sample of a fifth of the time
    dt1, n1, nbytes1, toks1 = oracle_sample_run(b, budget_s / 5, orc, num_threads=1)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": orc.max_threads(),
            "kind": "oracle",
            "sample": f"oracle decode (fp64, OpenMP) of the first {n} of {b.num_seqs} sequences "
                      f"({toks} attended tokens), one run of {dt:.2f} s",
            "attended_tokens_per_s": round(toks / dt, 1),
            "one_thread": {"value": round(nbytes1 / dt1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                           "sample": f"the first {n1} sequences ({toks1} attended tokens), one run "
                                     f"of {dt1:.2f} s"}}


def cpu_baseline_fp8(b: W.PagedBatch, kc8, vc8, ks, vs, budget_s: float = 10.0):
    """The oracle's decode over the FP8 pool (codes copied from the device), first n sequences."""
    import oracle

    orc = oracle.load()
    n = 1
    while True:
        sub = W.sub_batch(b, np.arange(n))
        t0 = time.perf_counter()
        orc.decode(sub["query"], kc8, vc8, sub["block_tables"], sub["context_lens"], b.scale,
                   "fp8", q_dtype=b.dtype, k_scale=ks, v_scale=vs)
        dt = time.perf_counter() - t0
        if dt >= budget_s or n == b.num_seqs:
            break
        n = min(b.num_seqs, max(n + 1, int(n * min(8.0, budget_s / max(dt, 1e-4)))))
    sb = W.PagedBatch(**{**b.__dict__, "query": sub["query"], "block_tables": sub["block_tables"],
                          "context_lens": sub["context_lens"]})
    nbytes = decode_bytes(sb, ELT[b.dtype], unique=False, kv_elt=1)
    toks = int(sub["context_lens"].sum())
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": orc.max_threads(),
            "kind": "oracle",
            "sample": f"oracle decode over the FP8 pool (fp64, OpenMP) of the first {n} of "
                      f"{b.num_seqs} sequences ({toks} attended tokens), one run of {dt:.2f} s",
            "attended_tokens_per_s": round(toks / dt, 1)}


def cpu_baseline_prefill(b: W.PagedBatch, budget_s: float = 10.0):
    """The oracle's prefill of the first n sequences (their new tokens' rows)."""
    import oracle

    orc = oracle.load()
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    orc.reshape_and_cache(b.key, b.value, kc, vc, b.slot_mapping, b.dtype)
    qs = b.query_start
    n = 1
    while True:
        t0 = time.perf_counter()
        orc.prefill(b.query[:qs[n]], kc, vc, b.block_tables[:n], b.context_lens[:n], qs[:n + 1],
                    b.scale, b.dtype)
        dt = time.perf_counter() - t0
        if dt >= budget_s or n == b.num_seqs:
            break
        n = min(b.num_seqs, max(n + 1, int(n * min(8.0, budget_s / max(dt, 1e-4)))))
    sb = W.PagedBatch(**{**b.__dict__, "context_lens": b.context_lens[:n], "query_start": qs[:n + 1]})
    flops = prefill_flops(sb)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": orc.max_threads(),
            "kind": "oracle",
            "sample": f"oracle prefill (fp64, OpenMP) of the first {n} of {b.num_seqs} sequences "
                      f"({int(qs[n])} new tokens), one run of {dt:.2f} s",
            "new_tokens_per_s": round(int(qs[n]) / dt, 1)}


def run_reference_prefill(args, b: W.PagedBatch, config: dict):
    """The reference arm of a prefill workload: the oracle's cache write and prefill of the
    first n sequences per step, n sized so the whole run takes about two minutes."""
    import oracle

    orc = oracle.load()
    steps, warmup = args.steps, args.warmup
    per_step = max(0.005, 120.0 / max(1, steps + warmup))
    qs = b.query_start
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    n = 1
    while True:
        t0 = time.perf_counter()
        orc.prefill(b.query[:qs[n]], kc, vc, b.block_tables[:n], b.context_lens[:n], qs[:n + 1],
                    b.scale, b.dtype)
        dt = time.perf_counter() - t0
        if dt >= per_step or n == b.num_seqs:
            break
        n = min(b.num_seqs, max(n + 1, int(n * min(8.0, per_step / max(dt, 1e-4)))))

    def step():
        orc.reshape_and_cache(b.key[:qs[n]], b.value[:qs[n]], kc, vc, b.slot_mapping[:qs[n]], b.dtype)
        orc.prefill(b.query[:qs[n]], kc, vc, b.block_tables[:n], b.context_lens[:n], qs[:n + 1],
                    b.scale, b.dtype)

    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = (time.perf_counter() - t0) / max(1, steps)
    sb = W.PagedBatch(**{**b.__dict__, "context_lens": b.context_lens[:n], "query_start": qs[:n + 1]})
    value = prefill_flops(sb) / dt / 1e12
    line = {"impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": warmup, "ms_per_step": round(dt * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "new_tokens_per_s": round(int(qs[n]) / dt, 1),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": orc.max_threads(),
                             "kind": "oracle",
                             "sample": f"each step: oracle cache write + prefill of the first {n} of "
                                       f"{b.num_seqs} sequences ({int(qs[n])} new tokens)"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_fp8(args, b: W.PagedBatch, config: dict):
    """The reference arm of `--kv fp8`: the workload's pool quantised by the oracle with the
    same per-kv-head scales as the CUDA arm (largest magnitude of the head's rows / 240), then
    per step the oracle's FP8 cache write and decode of the first n sequences."""
    import oracle

    orc = oracle.load()
    steps, warmup = args.steps, args.warmup
    bs = b.block_size
    used = []
    for s in range(b.num_seqs):
        t = np.arange(max(int(b.context_lens[s]) - 1, 0))
        used.append(b.block_tables[s, t // bs].astype(np.int64) * bs + t % bs)
    used = np.unique(np.concatenate(used))
    rows_k = b.key_cache[used // bs, :, used % bs, :]
    rows_v = b.value_cache[used // bs, :, used % bs, :]

    def head_scales(rows, new):
        x = W.decode_to_f64(np.concatenate([rows, new]), b.dtype)
        return np.maximum(np.abs(x).max(axis=(0, 2)) / 240.0, 1e-8).astype(np.float32)

    ks, vs = head_scales(rows_k, b.key), head_scales(rows_v, b.value)
    kc8 = np.full(b.key_cache.shape, 0x7f, dtype=np.uint8)
    vc8 = np.full(b.value_cache.shape, 0x7f, dtype=np.uint8)
    orc.reshape_and_cache_fp8(rows_k, rows_v, b.dtype, kc8, vc8, used, ks, vs)
    per_step = max(0.005, 120.0 / max(1, steps + warmup))
    n = 1
    while True:
        sub = W.sub_batch(b, np.arange(n))
        t0 = time.perf_counter()
        orc.decode(sub["query"], kc8, vc8, sub["block_tables"], sub["context_lens"], b.scale, "fp8",
                   q_dtype=b.dtype, k_scale=ks, v_scale=vs)
        dt = time.perf_counter() - t0
        if dt >= per_step or n == b.num_seqs:
            break
        n = min(b.num_seqs, max(n + 1, int(n * min(8.0, per_step / max(dt, 1e-4)))))

    def step():
        orc.reshape_and_cache_fp8(b.key[:n], b.value[:n], b.dtype, kc8, vc8, b.slot_mapping[:n], ks, vs)
        orc.decode(sub["query"], kc8, vc8, sub["block_tables"], sub["context_lens"], b.scale, "fp8",
                   q_dtype=b.dtype, k_scale=ks, v_scale=vs)

    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = (time.perf_counter() - t0) / max(1, steps)
    sb = W.PagedBatch(**{**b.__dict__, "query": sub["query"], "block_tables": sub["block_tables"],
                          "context_lens": sub["context_lens"]})
    step_bytes = (decode_bytes(sb, ELT[b.dtype], unique=False, kv_elt=1)
                  + n * b.num_kv_heads * b.head_dim * (ELT[b.dtype] + 1) * 2 + n * 8)
    value = step_bytes / dt / 1e9
    toks = int(sub["context_lens"].sum())
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": warmup, "ms_per_step": round(dt * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(config, kv_dtype="fp8_e4m3",
                                                kv_scales="per kv head: max |x| / 240"),
            "attended_tokens_per_s": round(toks / dt, 1),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": orc.max_threads(),
                             "kind": "oracle",
                             "sample": f"each step: oracle FP8 cache write + decode of the first {n} of "
                                       f"{b.num_seqs} sequences ({toks} attended tokens)"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_swap(args, b: W.PagedBatch, config: dict):
    """The reference arm of `--swap`: the oracle moves every block the batch uses from the
    pool to a second pool (scattered ids) and back, timed on the host."""
    import oracle

    orc = oracle.load()
    ids = []
    for s in range(b.num_seqs):
        ids.extend(b.block_tables[s, :-(-int(b.context_lens[s]) // b.block_size)].tolist())
    ids = np.array(sorted(set(ids)), np.int64)
    n = len(ids)
    rng = np.random.default_rng(0)
    host_ids = rng.permutation(n).astype(np.int64)
    hk = np.empty((n,) + b.key_cache.shape[1:], dtype=b.key_cache.dtype)
    hv = np.empty_like(hk)
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    out_pairs = np.stack([ids, host_ids], 1)
    in_pairs = np.stack([host_ids, rng.permutation(ids)], 1)
    block_bytes = int(np.prod(b.key_cache.shape[1:])) * ELT[b.dtype] * 2
    total = n * block_bytes

    def step():
        orc.swap_blocks(kc, vc, hk, hv, out_pairs, b.dtype)
        orc.swap_blocks(hk, hv, kc, vc, in_pairs, b.dtype)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    value = 2 * total / dt / 1e9  # both directions per step
    line = {"impl": "reference", "metric": "block swap GB/s (device <-> pinned host, pa_swap_blocks)",
            "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 4), "higher_is_better": True,
            "dtype": b.dtype, "data": "synthetic",
            "config": dict(config, swapped_blocks=n, bytes_per_direction=total),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step: all {n} blocks out and back, host memory"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference(args, b: W.PagedBatch, config: dict):
    if b.query_start is not None:
        return run_reference_prefill(args, b, config)
    if args.swap:
        return run_reference_swap(args, b, config)
    if args.kv == "fp8":
        return run_reference_fp8(args, b, config)
    import oracle

    orc = oracle.load()
    steps, warmup = args.steps, args.warmup
    # each step decodes a bounded sample, sized so the whole run takes about two minutes
    per_step = max(0.005, 120.0 / max(1, steps + warmup))
    _, n, nbytes, toks = oracle_sample_run(b, per_step, orc)
    sub = W.sub_batch(b, np.arange(n))
    kc, vc = b.key_cache.copy(), b.value_cache.copy()

    def step():
        orc.reshape_and_cache(b.key[:n], b.value[:n], kc, vc, b.slot_mapping[:n], b.dtype)
        orc.decode(sub["query"], kc, vc, sub["block_tables"], sub["context_lens"], b.scale, b.dtype)

    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = (time.perf_counter() - t0) / max(1, steps)
    e = ELT[b.dtype]
    step_bytes = nbytes + n * b.num_kv_heads * b.head_dim * e * 4 + n * 8
    value = step_bytes / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": warmup, "ms_per_step": round(dt * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "attended_tokens_per_s": round(toks / dt, 1),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": orc.max_threads(),
                             "kind": "oracle",
                             "sample": f"each step: oracle cache write + decode of the first {n} of "
                                       f"{b.num_seqs} sequences ({toks} attended tokens)"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------------------------

def make_batch(name: str) -> W.PagedBatch:
    return W.workload(name)


def max_over_ranks(vals, device=None) -> list:
    """Element-wise maximum of `vals` over the ranks of the default process group (each rank's
    times: the slowest rank's count); the values unchanged outside a multi-rank group."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def run_ours(args, b: W.PagedBatch, config: dict, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import paged_kv_cache_427_b200 as pa

    pa.load()
    dev = torch.device("cuda", local_rank)
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[b.dtype]
    out_dtype = tdt

    def dev_t(a, dt=None):
        if dt == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    # rotating pools: enough copies that each step's attended bytes push the previous step's
    # rows out of L2 before they are read again
    att = attended_bytes(b)
    rot = args.rotations or max(2, min(8, math.ceil(3 * L2_BYTES / max(att, 1)) + 1))
    kc0 = dev_t(b.key_cache, b.dtype)
    vc0 = dev_t(b.value_cache, b.dtype)
    pools = [(kc0, vc0)] + [(kc0.clone(), vc0.clone()) for _ in range(rot - 1)]
    q = dev_t(b.query, b.dtype)
    key = dev_t(b.key, b.dtype)
    value = dev_t(b.value, b.dtype)
    slots = dev_t(b.slot_mapping)
    tables = dev_t(b.block_tables)
    lens = dev_t(b.context_lens)
    mapping = dev_t(b.block_mapping) if b.block_mapping is not None and len(b.block_mapping) else None
    out = torch.empty(q.shape, dtype=out_dtype, device=dev)
    stream = torch.cuda.current_stream()
    ws = None
    if args.decode_flags:
        ws = torch.zeros(pa.pa_decode_workspace_bytes(b.num_seqs, b.num_heads, b.num_kv_heads,
                                                      b.head_dim, 0), dtype=torch.uint8, device=dev)

    def decode(qq, kc, vc, tt, ll):
        if ws is None:
            pa.pa_decode(out, qq, kc, vc, tt, ll, b.scale, b.block_size, b.num_kv_heads)
        else:
            pa.pa_decode_ex(out, qq, kc, vc, tt, ll, b.scale, b.block_size, b.num_kv_heads,
                            flags=args.decode_flags, workspace=ws)

    def step(i, ev=None):
        kc, vc = pools[i % rot]
        if mapping is not None:
            pa.pa_copy_blocks(kc, vc, mapping)
        pa.pa_reshape_and_cache(key, value, kc, vc, slots)
        if ev is not None:
            ev[0].record(stream)
        decode(q, kc, vc, tables, lens)
        if ev is not None:
            ev[1].record(stream)

    launches_per_step = 2 + (1 if mapping is not None else 0) + (1 if args.decode_flags & 1 else 0)
    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        pass
    sampler = ClockSampler(gpu_uuid).start()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    # a short soak so the clock sampler sees the GPU under this load even when K is small
    t_soak = time.perf_counter()
    i = 0
    while time.perf_counter() - t_soak < args.soak:
        for _ in range(200):
            step(i)
            i += 1
        torch.cuda.synchronize()

    # Timed region 1: K whole steps with nothing between the launches, so each decode may
    # start while the write before it finishes (programmatic dependent launch).
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed_ms = start.elapsed_time(end)
    # Timed region 2: the same K steps with a CUDA event pair around every decode launch (an
    # event between the write and the decode serialises them), for the decode kernel's own
    # duration in the roofline.
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        step(i, evs[i])
    torch.cuda.synchronize()
    decode_ms = [s.elapsed_time(e) for s, e in evs]

    # Timed region 3 (default flags only): the step as one pa_decode_step call, captured once
    # per pool copy into a CUDA graph and replayed K times.
    graph = None
    if args.decode_flags == pa.PA_DECODE_OVERLAP_PREVIOUS and world == 1:
        def graph_step(i):
            kc, vc = pools[i % rot]
            if mapping is not None:
                pa.pa_copy_blocks(kc, vc, mapping)
            pa.pa_decode_step(key, value, kc, vc, slots, out, q, tables, lens, b.scale,
                              b.block_size, b.num_kv_heads, workspace=ws)
        for i in range(rot):
            graph_step(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(rot):
                graph_step(i)
        reps = max(1, args.steps // rot)
        for _ in range(3):
            g.replay()
        g_start, g_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        g_start.record(stream)
        for _ in range(reps):
            g.replay()
        g_end.record(stream)
        torch.cuda.synchronize()
        graph = (g_start.elapsed_time(g_end) / (reps * rot), reps * rot)
        del g

    # end to end through the same calls: inputs from pinned host memory, output read back
    def host_t(a, dt=None):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16) if dt == "bf16" else a)
        return (t.view(torch.bfloat16) if dt == "bf16" else t).pin_memory()

    # One pinned host buffer holds every input of the step (each piece 256-byte aligned); one
    # copy brings it to the device, where the calls read views of it.
    parts = {"query": host_t(b.query, b.dtype), "key": host_t(b.key, b.dtype),
             "value": host_t(b.value, b.dtype), "slots": host_t(b.slot_mapping),
             "tables": host_t(b.block_tables), "lens": host_t(b.context_lens)}
    if mapping is not None:
        parts["mapping"] = host_t(b.block_mapping)
    offs, total = {}, 0
    for k, t in parts.items():
        offs[k] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_buf = torch.empty(total, dtype=torch.uint8).pin_memory()
    for k, t in parts.items():
        n = t.numel() * t.element_size()
        h_buf[offs[k]:offs[k] + n].copy_(t.reshape(-1).view(torch.uint8))
    d_buf = torch.empty(total, dtype=torch.uint8, device=dev)

    def dview(k):
        t = parts[k]
        n = t.numel() * t.element_size()
        return d_buf[offs[k]:offs[k] + n].view(t.dtype).view(t.shape)

    d_in = {k: dview(k) for k in parts}
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = total
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step(i):
        d_buf.copy_(h_buf, non_blocking=True)
        kc, vc = pools[i % rot]
        if mapping is not None:
            pa.pa_copy_blocks(kc, vc, d_in["mapping"])
        pa.pa_reshape_and_cache(d_in["key"], d_in["value"], kc, vc, d_in["slots"])
        decode(d_in["query"], kc, vc, d_in["tables"], d_in["lens"])
        h_out.copy_(out, non_blocking=True)
        stream.synchronize()

    e2e_steps = args.steps
    for i in range(min(args.warmup, 50)):
        e2e_step(i)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    e_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_start.elapsed_time(e_end)

    # The same end-to-end step with its four operations (input copy, pa_decode_step or its two
    # halves, output copy) captured in one CUDA graph per pool copy: one launch per step, still
    # a synchronize and a host read of the output every step.
    e2e_graph_ms = None
    if args.decode_flags == pa.PA_DECODE_OVERLAP_PREVIOUS and world == 1:
        def e2e_body(i):
            d_buf.copy_(h_buf, non_blocking=True)
            kc, vc = pools[i % rot]
            if mapping is not None:
                pa.pa_copy_blocks(kc, vc, d_in["mapping"])
            pa.pa_decode_step(d_in["key"], d_in["value"], kc, vc, d_in["slots"], out,
                              d_in["query"], d_in["tables"], d_in["lens"], b.scale, b.block_size,
                              b.num_kv_heads, workspace=ws)
            h_out.copy_(out, non_blocking=True)
        graphs = []
        for j in range(rot):
            e2e_body(j)
            torch.cuda.synchronize()
            gj = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gj):
                e2e_body(j)
            graphs.append(gj)
        for i in range(min(args.warmup, 50)):
            graphs[i % rot].replay()
            stream.synchronize()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for i in range(e2e_steps):
            graphs[i % rot].replay()
            stream.synchronize()
        g1.record(stream)
        torch.cuda.synchronize()
        e2e_graph_ms = g0.elapsed_time(g1)
        del graphs
    clocks = sampler.stop()

    elapsed_ms, e2e_ms, dec_mean = max_over_ranks([elapsed_ms, e2e_ms, float(np.mean(decode_ms))],
                                                  device=dev)
    flags = pa.pa_get_device_error(clear=True)
    if rank != 0:
        return
    if flags:
        print(f"warning: device error word 0x{flags:x}", file=sys.stderr)

    out_elt = torch.tensor([], dtype=out_dtype).element_size()
    dec_unique = decode_bytes(b, out_elt, unique=True)
    dec_logical = decode_bytes(b, out_elt, unique=False)
    step_bytes = dec_unique + write_bytes(b)
    ms = elapsed_ms / args.steps
    value = world * step_bytes / (ms * 1e-3) / 1e9
    e2e_ms_step = e2e_ms / e2e_steps
    peak, peak_src = hbm_peak()
    achieved = dec_unique / (dec_mean * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": b.dtype,
        "data": "synthetic", "config": config,
        "attended_tokens_per_s": round(world * b.attended_tokens / (ms * 1e-3), 1),
        "seq_steps_per_s": round(world * b.num_seqs / (ms * 1e-3), 1),
        "pct_of_8TBs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        f"pct_of_{peak_src}_hbm": round(100 * value / world / peak, 2),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": recorded_traffic(config["workload"]),
                     "kernel": ("paged_decode_kernel (CUDA cores)"
                                if (args.decode_flags & 2 or b.dtype == "f32")
                                else "paged_decode_mma_kernel (mma.sync + TMA)"),
                     "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": dec_unique,
                     "mean_launch_us": round(dec_mean * 1e3, 3),
                     "launch_timing": "CUDA events around each decode launch, in a second timed "
                                      "region of the same K steps"},
        "e2e": {"value": round(world * step_bytes / (e2e_ms_step * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "ms_per_step": round(e2e_ms_step, 5),
                "how": "per step: one pinned-buffer copy in, the write, the decode, the output "
                       "copy out, synchronize"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if e2e_graph_ms is not None:
        g_step = e2e_graph_ms / e2e_steps
        line["e2e_graph"] = {"value": round(step_bytes / (g_step * 1e-3) / 1e9, 2), "unit": "GB/s",
                             "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                             "ms_per_step": round(g_step, 5),
                             "how": "the same four operations per step captured in one CUDA "
                                    "graph (per pool copy), replayed, synchronize every step"}
    if graph is not None:
        line["graph"] = {"ms_per_step": round(graph[0], 5),
                         "value": round(step_bytes / (graph[0] * 1e-3) / 1e9, 2), "unit": "GB/s",
                         "steps": graph[1],
                         "how": "pa_decode_step (+ pa_copy_blocks) captured in one CUDA graph per "
                                "pool copy, replayed"}
    if dec_logical != dec_unique:
        line["logical_GBps"] = round(world * (dec_logical + write_bytes(b)) / (ms * 1e-3) / 1e9, 2)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(b, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_fp8(args, b, config):
    """The same decode step over an FP8 E4M3 cache: the pool is the workload's pool quantised
    (per-kv-head scales: largest magnitude of the head's rows / 240), each step writes the new
    tokens with pa_reshape_and_cache_fp8 and decodes with pa_decode_fp8 launched to overlap the
    write.  Timed like the 16-bit step: K steps with nothing between launches (`value`), then
    the same K steps with events around each decode (the roofline)."""
    import torch

    import paged_kv_cache_427_b200 as pa

    pa.load()
    dev = torch.device("cuda", 0)
    FP8 = torch.float8_e4m3fn

    def dev_t(a, dt=None):
        if dt == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    kc16, vc16 = dev_t(b.key_cache, b.dtype), dev_t(b.value_cache, b.dtype)
    # every slot the step's contexts use, except the new tokens' (the step writes those)
    used = []
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        t = np.arange(max(L - 1, 0))
        used.append(b.block_tables[s, t // b.block_size].astype(np.int64) * b.block_size
                    + t % b.block_size)
    used = np.unique(np.concatenate(used))
    su = torch.from_numpy(used).to(dev)
    rows_k = kc16[su // b.block_size, :, su % b.block_size, :].contiguous()  # [n, Hkv, D]
    rows_v = vc16[su // b.block_size, :, su % b.block_size, :].contiguous()
    key, value = dev_t(b.key, b.dtype), dev_t(b.value, b.dtype)
    ks = (torch.cat([rows_k, key]).float().abs().amax(dim=(0, 2)) / 240.0).clamp_min(1e-8).contiguous()
    vs = (torch.cat([rows_v, value]).float().abs().amax(dim=(0, 2)) / 240.0).clamp_min(1e-8).contiguous()
    att = attended_bytes(b) // 2
    rot = args.rotations or max(2, min(8, math.ceil(3 * L2_BYTES / max(att, 1)) + 1))
    pools = []
    for _ in range(rot):
        kc = torch.full(kc16.shape, 0x7f, dtype=torch.uint8, device=dev).view(FP8)
        vc = torch.full(vc16.shape, 0x7f, dtype=torch.uint8, device=dev).view(FP8)
        pa.pa_reshape_and_cache_fp8(rows_k, rows_v, kc, vc, su, ks, vs)
        pools.append((kc, vc))
    del kc16, vc16, rows_k, rows_v
    q = dev_t(b.query, b.dtype)
    slots, tables, lens = dev_t(b.slot_mapping), dev_t(b.block_tables), dev_t(b.context_lens)
    out = torch.empty(q.shape, dtype=q.dtype, device=dev)
    ws = torch.zeros(pa.pa_decode_workspace_bytes(b.num_seqs, b.num_heads, b.num_kv_heads,
                                                  b.head_dim, 0), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, ev=None):
        kc, vc = pools[i % rot]
        pa.pa_reshape_and_cache_fp8(key, value, kc, vc, slots, ks, vs)
        if ev is not None:
            ev[0].record(stream)
        pa.pa_decode_fp8(out, q, kc, vc, tables, lens, ks, vs, b.scale, b.block_size,
                         b.num_kv_heads, 0, pa.PA_DECODE_OVERLAP_PREVIOUS, ws)
        if ev is not None:
            ev[1].record(stream)

    sampler = ClockSampler(None).start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    t_soak = time.perf_counter()
    i = 0
    while time.perf_counter() - t_soak < args.soak:
        for _ in range(200):
            step(i)
            i += 1
        torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    elapsed_ms = start.elapsed_time(end)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        step(i, evs[i])
    torch.cuda.synchronize()
    dec_mean = float(np.mean([s_.elapsed_time(e_) for s_, e_ in evs]))
    clocks = sampler.stop()
    flags = pa.pa_get_device_error(clear=True)
    if flags:
        print(f"warning: device error word 0x{flags:x}", file=sys.stderr)
    dec = decode_bytes(b, ELT[b.dtype], unique=True, kv_elt=1)
    t_new = int((b.slot_mapping >= 0).sum())
    wbytes = t_new * b.num_kv_heads * b.head_dim * (ELT[b.dtype] + 1) * 2 + len(b.slot_mapping) * 8
    ms = elapsed_ms / args.steps
    value = (dec + wbytes) / (ms * 1e-3) / 1e9
    peak, peak_src = hbm_peak()
    achieved = dec / (dec_mean * 1e-3) / 1e9
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3 cache, bf16 query", "data": "synthetic",
            "config": dict(config, kv_dtype="fp8_e4m3", pool_rotations=rot,
                           kv_scales="per kv head: max |x| / 240"),
            "attended_tokens_per_s": round(b.attended_tokens / (ms * 1e-3), 1),
            "seq_steps_per_s": round(b.num_seqs / (ms * 1e-3), 1),
            "pct_of_8TBs": round(100 * value / NOMINAL_HBM_GBS, 2),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                         "kernel": "paged_decode_mma_kernel (fp8 e4m3 cache)",
                         "peak_source": peak_src, "algorithmic_bytes_per_launch": dec,
                         "mean_launch_us": round(dec_mean * 1e3, 3),
                         "launch_timing": "CUDA events around each decode launch, in a second "
                                          "timed region of the same K steps"},
            "gpu_launches": 2 * args.steps, "clocks": clocks}
    if not args.no_cpu_baseline:
        kc8, vc8 = pools[0]
        line["cpu_baseline"] = cpu_baseline_fp8(
            b, kc8.view(torch.uint8).cpu().numpy(), vc8.view(torch.uint8).cpu().numpy(),
            ks.cpu().numpy(), vs.cpu().numpy(), args.cpu_seconds)
    print(json.dumps(line), flush=True)


def prefill_flops(b: W.PagedBatch) -> int:
    """Algorithmic FLOPs of a prefill step: each new token's row of each query head takes
    2*D FLOPs per attended position for q.K and 2*D for P.V (causal: positions 0 .. p)."""
    qs = b.query_start
    tot = 0
    for s in range(b.num_seqs):
        L, q = int(b.context_lens[s]), int(qs[s + 1] - qs[s])
        p = np.arange(L - q, L, dtype=np.int64)
        tot += int((p + 1).sum())
    return 4 * b.head_dim * b.num_heads * tot


def run_prefill(args, b, config):
    """A chunked-prefill step: the new tokens' K/V written (pa_reshape_and_cache), then
    pa_prefill.  Timed like the decode step; the roofline is tensor-bound, against the measured
    bf16 dense GEMM rate (the burst figure: the kernel is timed alone per launch)."""
    import torch

    import paged_kv_cache_427_b200 as pa

    pa.load()
    dev = torch.device("cuda", 0)

    def dev_t(a, dt=None):
        if dt == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    kc0, vc0 = dev_t(b.key_cache, b.dtype), dev_t(b.value_cache, b.dtype)
    att = attended_bytes(b)
    rot = args.rotations or max(2, min(8, math.ceil(3 * L2_BYTES / max(att, 1)) + 1))
    pools = [(kc0, vc0)] + [(kc0.clone(), vc0.clone()) for _ in range(rot - 1)]
    q = dev_t(b.query, b.dtype)
    key, value = dev_t(b.key, b.dtype), dev_t(b.value, b.dtype)
    slots, tables = dev_t(b.slot_mapping), dev_t(b.block_tables)
    lens, qs = dev_t(b.context_lens), dev_t(b.query_start)
    out = torch.empty(q.shape, dtype=q.dtype, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, ev=None):
        kc, vc = pools[i % rot]
        pa.pa_reshape_and_cache(key, value, kc, vc, slots)
        if ev is not None:
            ev[0].record(stream)
        pa.pa_prefill(out, q, kc, vc, tables, lens, qs, b.scale, b.block_size, b.num_kv_heads)
        if ev is not None:
            ev[1].record(stream)

    sampler = ClockSampler(None).start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    t_soak = time.perf_counter()
    i = 0
    while time.perf_counter() - t_soak < args.soak:
        for _ in range(50):
            step(i)
            i += 1
        torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    elapsed_ms = start.elapsed_time(end)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        step(i, evs[i])
    torch.cuda.synchronize()
    k_ms = float(np.mean([s_.elapsed_time(e_) for s_, e_ in evs]))
    clocks = sampler.stop()
    flags = pa.pa_get_device_error(clear=True)
    if flags:
        print(f"warning: device error word 0x{flags:x}", file=sys.stderr)
    flops = prefill_flops(b)
    ms = elapsed_ms / args.steps
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        peak, src = 1590.0, "fallback"
    tflops = flops / (k_ms * 1e-3) / 1e12
    new_tokens = int(b.query_start[-1])
    line = {"metric": PREFILL_METRIC, "value": round(flops / (ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": b.dtype, "data": "synthetic",
            "config": dict(config, new_tokens=new_tokens, pool_rotations=rot,
                           query_lens=[int(x) for x in np.diff(b.query_start)]),
            "new_tokens_per_s": round(new_tokens / (ms * 1e-3), 1),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "traffic": None,
                         "kernel": "paged_prefill_tc_kernel (tcgen05 + TMEM + TMA)", "peak_source": src,
                         "algorithmic_flops_per_launch": flops,
                         "mean_launch_us": round(k_ms * 1e3, 3)},
            "gpu_launches": 2 * args.steps, "clocks": clocks}
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(b, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_swap(args, b, config):
    """Block swap between the device cache and a pinned host cache: every block the batch's
    sequences use goes out (device -> host, scattered host ids) and back in (host -> device,
    scattered device ids), each direction one pa_swap_blocks call timed with CUDA events.  The
    roofline is the host link as one plain cudaMemcpyAsync of the same bytes between one
    contiguous pinned buffer and device memory moves them, measured in the same run."""
    import torch

    import paged_kv_cache_427_b200 as pa

    pa.load()
    dev = torch.device("cuda", 0)
    t = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[b.dtype]

    def dev_t(a, dt=None):
        if dt == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    kc, vc = dev_t(b.key_cache, b.dtype), dev_t(b.value_cache, b.dtype)
    ids = []
    for s in range(b.num_seqs):
        ids.extend(b.block_tables[s, :-(-int(b.context_lens[s]) // b.block_size)].tolist())
    ids = np.array(sorted(set(ids)), np.int64)
    n = len(ids)
    rng = np.random.default_rng(0)
    host_ids = rng.permutation(n).astype(np.int64)
    hk = torch.empty((n,) + tuple(kc.shape[1:]), dtype=t).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.from_numpy(np.stack([ids, host_ids], 1)).to(dev)
    in_pairs = torch.from_numpy(np.stack([host_ids, rng.permutation(ids)], 1)).to(dev)
    block_bytes = kc[0].numel() * kc.element_size() * 2  # K and V of one block
    total = n * block_bytes
    flat_h = torch.empty(total, dtype=torch.uint8).pin_memory()
    flat_d = torch.empty(total, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    reps = max(3, min(args.steps, 50))
    out_ms = timed(lambda: pa.pa_swap_blocks(kc, vc, hk, hv, out_pairs), reps)
    in_ms = timed(lambda: pa.pa_swap_blocks(hk, hv, kc, vc, in_pairs), reps)
    d2h_ms = timed(lambda: flat_h.copy_(flat_d, non_blocking=True), reps)
    h2d_ms = timed(lambda: flat_d.copy_(flat_h, non_blocking=True), reps)
    gbs = lambda ms: total / (ms * 1e-3) / 1e9
    flags = pa.pa_get_device_error(clear=True)
    if flags:
        print(f"warning: device error word 0x{flags:x}", file=sys.stderr)
    line = {"metric": "block swap GB/s (device <-> pinned host, pa_swap_blocks)",
            "value": round(gbs((out_ms + in_ms) / 2), 2), "unit": "GB/s", "n_gpus": 1,
            "steps": reps, "warmup": args.warmup, "higher_is_better": True,
            "dtype": b.dtype, "data": "synthetic",
            "config": dict(config, swapped_blocks=n, bytes_per_direction=total),
            "swap_out": {"ms": round(out_ms, 4), "GBps": round(gbs(out_ms), 2),
                         "link_GBps": round(gbs(d2h_ms), 2), "frac": round(d2h_ms / out_ms, 4)},
            "swap_in": {"ms": round(in_ms, 4), "GBps": round(gbs(in_ms), 2),
                        "link_GBps": round(gbs(h2d_ms), 2), "frac": round(h2d_ms / in_ms, 4)},
            "roofline": {"bound": "host link", "peak_source": "cudaMemcpyAsync of one contiguous "
                         "pinned buffer of the same bytes, same run"},
            "gpu_launches": 2 * reps}
    if not args.no_cpu_baseline:
        import oracle

        orc = oracle.load()
        hk_o = np.empty((n,) + b.key_cache.shape[1:], dtype=b.key_cache.dtype)
        hv_o = np.empty_like(hk_o)
        pairs = np.stack([ids, host_ids], 1)
        t0, k = time.perf_counter(), 0
        while time.perf_counter() - t0 < min(args.cpu_seconds, 5.0) or k == 0:
            orc.swap_blocks(b.key_cache, b.value_cache, hk_o, hv_o, pairs, b.dtype)
            k += 1
        dt = (time.perf_counter() - t0) / k
        line["cpu_baseline"] = {"value": round(total / dt / 1e9, 4), "unit": "GB/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"oracle swap-out of the same {n} blocks (host memory to "
                                          f"host memory), {k} runs"}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="llama3_8b_decode",
                    help="llama3_8b_decode | short_chat_bs{8,16,32} | shared_prefix | long_mixed | "
                         "tiny_fp32 | chunked_prefill (pa_prefill)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-flags", type=int, default=4,
                    help="pa_decode_ex flags: 4 = start while the cache write runs (default), "
                         "2 = CUDA-core kernel, 1 = separate merge kernel, 0 = plain pa_decode")
    ap.add_argument("--rotations", type=int, default=0, help="copies of the KV pool (0 = enough to defeat L2)")
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of untimed load for the clock sampler")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv", default="native", choices=["native", "fp8"],
                    help="fp8: the same step over an FP8 E4M3 cache (pa_decode_fp8)")
    ap.add_argument("--swap", action="store_true",
                    help="measure block swap (pa_swap_blocks) of the workload's blocks instead")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        args.gpus = world if world > 1 else args.gpus
    b = make_batch(args.workload)
    config = {"workload": args.workload, "num_seqs": b.num_seqs, "num_heads": b.num_heads,
              "num_kv_heads": b.num_kv_heads, "head_dim": b.head_dim, "block_size": b.block_size,
              "kv_dtype": b.dtype, "attended_tokens": b.attended_tokens,
              "num_blocks": b.num_blocks, "max_blocks_per_seq": b.max_blocks,
              "seed": b.meta.get("seed"),
              "l2": "inputs larger than L2: steps rotate over copies of the KV pool",
              "pool_rotations": args.rotations or "auto",
              "decode_flags": args.decode_flags,
              "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, b, config)
        return

    import torch

    torch.cuda.set_device(local_rank)
    if args.swap:
        if rank == 0:
            run_swap(args, b, config)
        return
    if args.kv == "fp8":
        if rank == 0:
            run_fp8(args, b, config)
        return
    if b.query_start is not None:
        if rank == 0:
            run_prefill(args, b, config)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, b, config, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
