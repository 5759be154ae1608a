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


def bf16_peak():
    """Dense bf16 tensor rate: the burst figure (a kernel timed alone per launch)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


# The files each kernel's device code is compiled from (its traffic record is void once any
# of them changes).
KERNEL_SOURCES = {
    "decode": ("pa_decode_mma.cuh", "pa_decode_common.cuh", "pa_decode.cuh", "pa_device.cuh",
               "pa_internal.h", "pa_decode_bf16_d128.cu"),
    "decode_fp8": ("pa_decode_mma.cuh", "pa_decode_common.cuh", "pa_decode.cuh", "pa_device.cuh",
                   "pa_internal.h", "pa_decode_fp8_bf16q.cu"),
    "prefill": ("pa_prefill_tc.cuh", "pa_tc.cuh", "pa_device.cuh", "pa_prefill_internal.h",
                "pa_prefill_bf16.cu"),
}
# the shared-prefix cascade: the prefill kernel's prefix pass and the decode kernel
KERNEL_SOURCES["shared"] = tuple(sorted(set(KERNEL_SOURCES["decode"]) | set(KERNEL_SOURCES["prefill"])))


def kernel_sources_digest(kernel: str = "decode") -> str:
    """Digest of the files a kernel is compiled from (device code and its argument block),
    not the host-side API or the other kernels."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_427_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f in KERNEL_SOURCES[kernel]:
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(key: str, kernel: str = "decode"):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json, keyed by
    workload, ':fp8' for the FP8 cache), if it was taken on the current kernel sources; else
    None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        entry = rec.get(key)
        if entry and entry.get("sources") == kernel_sources_digest(kernel):
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
    return dt, n, decode_bytes(sb, ELT[b.dtype], unique=True), int(sub["context_lens"].sum())


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
    nbytes = decode_bytes(sb, ELT[b.dtype], unique=True, kv_elt=1)
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
    step_bytes = (decode_bytes(sb, ELT[b.dtype], unique=True, kv_elt=1)
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


# ----------------------------------------------------------------------------------------------
# timing helpers
# ----------------------------------------------------------------------------------------------

def launch_stats(ms) -> dict:
    """Mean, median and minimum of per-launch CUDA-event durations (ms in, us out)."""
    us = np.asarray(ms, dtype=np.float64) * 1e3
    return {"mean_launch_us": round(float(us.mean()), 3),
            "median_launch_us": round(float(np.median(us)), 3),
            "min_launch_us": round(float(us.min()), 3), "launches": int(us.size)}


def launch_count(args) -> int:
    """Launches timed one by one for the roofline: at least 50, at most 500."""
    return max(50, min(args.steps, 500))


def pool_rotations(args, attended: int) -> int:
    """Copies of the KV pool that consecutive steps rotate over, enough that one step's
    attended bytes push the previous step's rows out of L2 before they are read again."""
    return args.rotations or max(2, min(8, math.ceil(3 * L2_BYTES / max(attended, 1)) + 1))


def dev_tensor(a, dt, dev):
    """Device tensor with the bytes of host array `a` (bf16 held as uint16 patterns)."""
    import torch

    a = np.ascontiguousarray(a)
    if dt == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(a).to(dev)


def run_steps(step, n: int, stream, first: int = 0) -> float:
    """n steps with nothing between the launches, one event pair around them: total ms."""
    import torch

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(first, first + n):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def run_launches(step, n: int) -> list:
    """n steps with an event pair around each step's main kernel: per-launch ms."""
    import torch

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    torch.cuda.synchronize()
    for i in range(n):
        step(i, evs[i])
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in evs]


def soak(step, seconds: float, per_round: int = 200):
    """Untimed load, so the clock sampler sees the GPU busy and clocks settle."""
    import torch

    t0, i = time.perf_counter(), 0
    while time.perf_counter() - t0 < seconds:
        for _ in range(per_round):
            step(i)
            i += 1
        torch.cuda.synchronize()


def hbm_roofline(alg_bytes: int, launch_ms, kernel: str, traffic, probe=None) -> dict:
    peak, src = hbm_peak()
    st = launch_stats(launch_ms)
    achieved = alg_bytes / (st["mean_launch_us"] * 1e-6) / 1e9
    r = {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
         "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kernel,
         "peak_source": src, "algorithmic_bytes_per_launch": int(alg_bytes), **st,
         "achieved_at_median": round(alg_bytes / (st["median_launch_us"] * 1e-6) / 1e9, 2),
         "launch_timing": "CUDA events around each launch on its stream, in a timed region of "
                          "its own after the step region"}
    if traffic:
        r["traffic_over_algorithmic"] = round(traffic / alg_bytes, 4)
    if probe:
        best = max(probe["ld_GBps"], probe["bulk_GBps"])
        r["read_probe_GBps"] = best
        r["frac_of_read_probe"] = round(achieved / best, 4)
    return r


def read_probe(dev, nbytes: int = 4 << 30, reps: int = 10) -> dict | None:
    """Read-only HBM bandwidth of this GPU: pa_hbm_read_probe over a buffer of `nbytes` (32x
    L2), both modes, median of `reps` launches after 3 warm-up launches."""
    import torch

    import paged_kv_cache_427_b200 as pa

    try:
        buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        buf.view(torch.int32).random_()
        sink = torch.zeros(4, dtype=torch.int32, device=dev)
        res = {}
        for mode, key in ((0, "ld_GBps"), (1, "bulk_GBps")):
            for _ in range(3):
                pa.pa_hbm_read_probe(buf, mode, sink)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(reps)]
            for e0, e1 in evs:
                e0.record()
                pa.pa_hbm_read_probe(buf, mode, sink)
                e1.record()
            torch.cuda.synchronize()
            ms = float(np.median([a.elapsed_time(b) for a, b in evs]))
            res[key] = round(nbytes / (ms * 1e-3) / 1e9, 1)
        if int(sink[1].item()) != 0:
            return None
        del buf
        torch.cuda.empty_cache()
        res.update({"bytes": nbytes, "reps": reps,
                    "how": "pa_hbm_read_probe: each byte read once; ld = 16-byte loads from 2048 "
                           "threads per SM, bulk = 32 KB bulk copies into a 6-slot shared-memory "
                           "ring per SM; median of the CUDA-event launch times"})
        return res
    except Exception as exc:  # the probe is evidence beside the numbers, never a reason to fail
        print(f"warning: read probe failed: {exc}", file=sys.stderr)
        return None


def timeline_summary(recs, chunk_bytes: int) -> dict:
    """Per-launch summary of decode timelines (pa_set_decode_timeline records, one array per
    launch), medians over the launches.  Times are us after the first worker warp started."""
    import paged_kv_cache_427_b200 as pa

    per = []
    sm_done = []
    for rec in recs:
        r = rec.reshape(-1, pa.TIMELINE_WORDS).astype(np.int64)
        r = r[r[:, pa.TL_START] > 0]  # warps of this launch
        live = r[:, pa.TL_CHUNKS] > 0
        if not live.any():
            continue
        o = r[:, pa.TL_START].min()
        us = lambda c: (r[live, c] - o) / 1e3  # noqa: E731
        done = np.maximum(r[live, pa.TL_DONE], r[live, pa.TL_MERGED]) - o
        done = done / 1e3
        first, last = us(pa.TL_FIRST), us(pa.TL_LAST)
        span = np.maximum(last - first, 1e-3)
        rates = r[live, pa.TL_CHUNKS] * chunk_bytes / (span * 1e-6) / 1e9
        end = float(done.max())
        per.append({"end_us": end,
                    "issue_us_p50": float(np.median(us(pa.TL_ISSUE))),
                    "first_tile_us_p10": float(np.percentile(first, 10)),
                    "first_tile_us_p50": float(np.median(first)),
                    "first_tile_us_p90": float(np.percentile(first, 90)),
                    "last_tile_us_p50": float(np.median(last)),
                    "done_us_p10": float(np.percentile(done, 10)),
                    "done_us_p50": float(np.median(done)),
                    "done_us_p90": float(np.percentile(done, 90)),
                    "tail_us": end - float(np.median(done)),
                    "sum_of_warp_rates_GBps": float(rates.sum())})
        sms = r[live, pa.TL_SM]
        d = {}
        for smv, dv in zip(sms, done):
            d[int(smv)] = max(d.get(int(smv), 0.0), float(dv))
        sm_done.append(d)
    if not per:
        return {}
    out = {k: round(float(np.median([p[k] for p in per])), 2) for k in per[0]}
    # do the same SMs finish last in every launch?  rank correlation of the SMs' finish times
    common = sorted(set.intersection(*[set(d) for d in sm_done])) if sm_done else []
    if len(sm_done) > 1 and len(common) > 2:
        ranks = [np.argsort(np.argsort([d[k] for k in common])) for d in sm_done]
        cs = [float(np.corrcoef(ranks[i], ranks[i + 1])[0, 1]) for i in range(len(ranks) - 1)]
        out["sm_finish_rank_corr"] = round(float(np.mean(cs)), 3)
        fin = np.array([[d[k] for k in common] for d in sm_done])
        out["sm_finish_us_min_p50_max"] = [round(float(x), 2) for x in
                                           (np.median(fin.min(1)), np.median(np.median(fin, 1)),
                                            np.median(fin.max(1)))]
    out["launches"] = len(per)
    out["how"] = ("pa_set_decode_timeline: globaltimer per worker warp at start, first tile "
                  "landed, last tile consumed, done (merges included); times after the first "
                  "warp started; medians over the launches")
    return out


# ----------------------------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------------------------

def run_decode(args, b: W.PagedBatch, config: dict, rank: int = 0, world: int = 1,
               local_rank: int = 0, full: bool = True, probe: dict | None = None,
               shared: bool = False) -> dict | None:
    """The decode step of one workload: the cache write (plus the copy-on-write block copies
    where the batch has them), then the decode launched to overlap the write.  Timed regions:
    K steps with nothing between launches (`value`); per-launch events around the decode (the
    roofline); with `full`, also the step as a CUDA graph, end to end from pinned host memory,
    the CPU baseline and the timeline.  With `shared`, the decode is pa_decode_shared_prefix
    over the batch's groups (workloads.shared_groups).  Returns rank 0's line (None on the
    other ranks)."""
    import torch

    import paged_kv_cache_427_b200 as pa

    pa.load()
    dev = torch.device("cuda", local_rank)
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[b.dtype]
    out_dtype = tdt

    rot = pool_rotations(args, attended_bytes(b))
    kc0 = dev_tensor(b.key_cache, b.dtype, dev)
    vc0 = dev_tensor(b.value_cache, b.dtype, dev)
    pools = [(kc0, vc0)] + [(kc0.clone(), vc0.clone()) for _ in range(rot - 1)]
    q = dev_tensor(b.query, b.dtype, dev)
    key = dev_tensor(b.key, b.dtype, dev)
    value = dev_tensor(b.value, b.dtype, dev)
    slots = dev_tensor(b.slot_mapping, None, dev)
    tables = dev_tensor(b.block_tables, None, dev)
    lens = dev_tensor(b.context_lens, None, dev)
    mapping = (dev_tensor(b.block_mapping, None, dev)
               if b.block_mapping is not None and len(b.block_mapping) else None)
    out = torch.empty(q.shape, dtype=out_dtype, device=dev)
    stream = torch.cuda.current_stream()
    ws = None
    if args.decode_flags:
        ws = torch.zeros(pa.pa_decode_workspace_bytes(b.num_seqs, b.num_heads, b.num_kv_heads,
                                                      b.head_dim, 0), dtype=torch.uint8, device=dev)

    if shared:
        g_start, p_lens = (dev_tensor(x, None, dev) for x in W.shared_groups(b))
        ws_shared = torch.zeros(pa.pa_decode_shared_prefix_workspace_bytes(
            b.num_seqs, b.num_heads, b.num_kv_heads, b.head_dim, b.max_blocks, b.block_size),
            dtype=torch.uint8, device=dev)

    def decode(qq, kc, vc, tt, ll, o=None):
        o = out if o is None else o
        if shared:
            pa.pa_decode_shared_prefix(o, qq, kc, vc, tt, ll, g_start, p_lens, b.scale,
                                       b.block_size, b.num_kv_heads, workspace=ws_shared)
        elif ws is None:
            pa.pa_decode(o, qq, kc, vc, tt, ll, b.scale, b.block_size, b.num_kv_heads)
        else:
            pa.pa_decode_ex(o, qq, kc, vc, tt, ll, b.scale, b.block_size, b.num_kv_heads,
                            flags=args.decode_flags, workspace=ws)

    # The whole step through pa_decode_step when the default flags apply (one kernel when each
    # sequence brings one new token: the write and the decode fused), else the write and the
    # decode as two calls.
    whole_step = (args.decode_flags == pa.PA_DECODE_OVERLAP_PREVIOUS and not shared
                  and b.dtype != "f32")
    fused = whole_step and len(b.slot_mapping) == b.num_seqs

    def step(i, ev=None):
        kc, vc = pools[i % rot]
        if mapping is not None:
            pa.pa_copy_blocks(kc, vc, mapping)
        if whole_step:
            if ev is not None:
                ev[0].record(stream)
            pa.pa_decode_step(key, value, kc, vc, slots, out, q, tables, lens, b.scale,
                              b.block_size, b.num_kv_heads, workspace=ws)
            if ev is not None:
                ev[1].record(stream)
            return
        pa.pa_reshape_and_cache(key, value, kc, vc, slots)
        if ev is not None:
            ev[0].record(stream)
        decode(q, kc, vc, tables, lens)
        if ev is not None:
            ev[1].record(stream)

    launches_per_step = ((1 if fused else 2) + (1 if mapping is not None else 0)
                         + (1 if args.decode_flags & 1 else 0) + (1 if shared else 0))
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
    soak(step, args.soak if full else min(args.soak, 0.3))

    # Timed region 1: K whole steps with nothing between the launches, so each decode may
    # start while the write before it finishes (programmatic dependent launch).
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    elapsed_ms = run_steps(step, args.steps, stream)
    if world > 1:
        dist.barrier()
    # Timed region 2: steps with a CUDA event pair around every decode launch (an event
    # between the write and the decode serialises them), for the decode kernel's own duration.
    decode_ms = run_launches(step, launch_count(args))

    # Timed region 3 (headline, default flags only): the step as one pa_decode_step call,
    # captured once per pool copy into a CUDA graph and replayed K times.
    graph = None
    if full and args.decode_flags == pa.PA_DECODE_OVERLAP_PREVIOUS and world == 1 and not shared:
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
        g_ms = run_steps(lambda i: g.replay(), reps, stream)
        graph = (g_ms / (reps * rot), reps * rot)
        del g

    e2e = None
    if full:
        e2e = measure_e2e(args, b, pools, rot, mapping, out, ws, decode, dev, stream, world)

    timeline = None
    if full and args.timeline and world == 1 and b.dtype != "f32" and not (args.decode_flags & 2):
        workers = pa.pa_decode_default_workers({"bf16": pa.PA_BF16, "f16": pa.PA_F16}[b.dtype],
                                               b.head_dim, b.block_size,
                                               b.num_heads // b.num_kv_heads)
        buf = torch.zeros(workers * pa.TIMELINE_WORDS, dtype=torch.int64, device=dev)
        pa.pa_set_decode_timeline(buf)
        recs = []
        try:
            for i in range(args.timeline):
                buf.zero_()
                step(i)
                torch.cuda.synchronize()
                recs.append(buf.cpu().numpy().copy())
        finally:
            pa.pa_set_decode_timeline(None)
        timeline = timeline_summary(recs, 16 * b.head_dim * ELT[b.dtype] * 2)
        if args.timeline_out:
            np.save(args.timeline_out, np.stack(recs))
    clocks = sampler.stop()

    elapsed_ms, dec_mean = max_over_ranks([elapsed_ms, float(np.mean(decode_ms))], device=dev)
    if e2e is not None:
        e2e["ms"], e2e["serial_ms"] = max_over_ranks([e2e["ms"], e2e["serial_ms"]], device=dev)
    flags = pa.pa_get_device_error(clear=True)
    if rank != 0:
        return None
    if flags:
        print(f"warning: device error word 0x{flags:x}", file=sys.stderr)

    out_elt = torch.tensor([], dtype=out_dtype).element_size()
    dec_unique = decode_bytes(b, out_elt, unique=True)
    dec_logical = decode_bytes(b, out_elt, unique=False)
    step_bytes = dec_unique + write_bytes(b)
    ms = elapsed_ms / args.steps
    value = world * step_bytes / (ms * 1e-3) / 1e9
    peak, peak_src = hbm_peak()
    kernel = ("paged_decode_kernel (CUDA cores)" if (args.decode_flags & 2 or b.dtype == "f32")
              else "paged_decode_mma_kernel (mma.sync + TMA)")
    if fused:
        kernel = ("paged_decode_mma_kernel (mma.sync + TMA), fused step: the cache write inside "
                  "the same kernel")
    roof_bytes = dec_unique + (write_bytes(b) if fused else 0)
    if shared:
        kernel = ("paged_prefill_tc_kernel shared-prefix pass (tcgen05) + paged_decode_mma_kernel "
                  "(mma.sync + TMA); launch times cover both")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": b.dtype,
        "data": "synthetic", "config": config,
        "attended_tokens_per_s": round(world * b.attended_tokens / (ms * 1e-3), 1),
        "seq_steps_per_s": round(world * b.num_seqs / (ms * 1e-3), 1),
        "pct_of_8TBs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        f"pct_of_{peak_src}_hbm": round(100 * value / world / peak, 2),
        "roofline": hbm_roofline(roof_bytes, decode_ms, kernel,
                                 recorded_traffic(config["workload"] + (":shared" if shared else ""),
                                                  "shared" if shared else "decode"), probe),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if probe:
        line["pct_of_read_probe"] = round(100 * value / world / max(probe["ld_GBps"], probe["bulk_GBps"]), 2)
    if e2e is not None:
        e_ms = e2e["ms"] / args.steps
        line["e2e"] = {"value": round(world * step_bytes / (e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                       "ms_per_step": round(e_ms, 5),
                       "how": "per step: one pinned-buffer copy of the step's inputs in (on a copy "
                              "stream, overlapping the previous step's compute; two buffers), the "
                              "write, the decode, the output copied out (on a second copy stream, "
                              "overlapping the next step's compute; two outputs) and waited for by "
                              "the host after the next step is launched"}
        s_ms = e2e["serial_ms"] / args.steps
        line["e2e_serial"] = {"value": round(world * step_bytes / (s_ms * 1e-3) / 1e9, 2),
                              "unit": "GB/s", "h2d_bytes_per_step": e2e["h2d"],
                              "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": round(s_ms, 5),
                              "how": "per step: the input copy, the write, the decode, the output "
                                     "copy, synchronize, nothing overlapped"}
        if e2e.get("graph_ms") is not None:
            g_step = e2e["graph_ms"] / args.steps
            line["e2e_graph"] = {"value": round(step_bytes / (g_step * 1e-3) / 1e9, 2),
                                 "unit": "GB/s", "h2d_bytes_per_step": e2e["h2d"],
                                 "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": round(g_step, 5),
                                 "how": "the same four operations per step captured in one CUDA "
                                        "graph (per pool copy), replayed, synchronize every step"}
        if e2e.get("breakdown"):
            line["e2e_breakdown"] = e2e["breakdown"]
    if graph is not None:
        line["graph"] = {"ms_per_step": round(graph[0], 5),
                         "value": round(step_bytes / (graph[0] * 1e-3) / 1e9, 2), "unit": "GB/s",
                         "steps": graph[1],
                         "how": "pa_decode_step (+ pa_copy_blocks) captured in one CUDA graph per "
                                "pool copy, replayed"}
    if dec_logical != dec_unique:
        line["logical_GBps"] = round(world * (dec_logical + write_bytes(b)) / (ms * 1e-3) / 1e9, 2)
    if timeline:
        line["timeline"] = timeline
    if shared:
        line["decode_call"] = "pa_decode_shared_prefix"
    elif whole_step:
        line["decode_call"] = "pa_decode_step" + (" (fused: one kernel)" if fused else "")
    if full and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(b, args.cpu_seconds)
    return line


def measure_e2e(args, b, pools, rot, mapping, out, ws, decode, dev, stream, world) -> dict:
    """The step end to end through the same public calls: every input of the step in one
    pinned host buffer, one copy in, the calls on device views of it, the output copied back and
    a synchronize, every step.  Also the same four operations captured in one CUDA graph per
    pool copy, and a per-operation breakdown of one eager step (events between the
    operations)."""
    import torch

    import paged_kv_cache_427_b200 as pa

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

    def e2e_step(i, ev=None):
        if ev is not None:
            ev[0].record(stream)
        d_buf.copy_(h_buf, non_blocking=True)
        if ev is not None:
            ev[1].record(stream)
        kc, vc = pools[i % rot]
        if mapping is not None:
            pa.pa_copy_blocks(kc, vc, d_in["mapping"])
        pa.pa_reshape_and_cache(d_in["key"], d_in["value"], kc, vc, d_in["slots"])
        if ev is not None:
            ev[2].record(stream)
        decode(d_in["query"], kc, vc, d_in["tables"], d_in["lens"])
        if ev is not None:
            ev[3].record(stream)
        h_out.copy_(out, non_blocking=True)
        if ev is not None:
            ev[4].record(stream)
        stream.synchronize()

    for i in range(min(args.warmup, 50)):
        e2e_step(i)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    res = {"serial_ms": e0.elapsed_time(e1), "h2d": int(total),
           "d2h": int(h_out.numel() * h_out.element_size())}

    # Pipelined, as a serving loop runs it: every step still copies its own inputs in and reads
    # its own result back, but step i's input copy runs on a copy stream while step i-1
    # computes (two input buffers, two outputs), step i-1's result goes back on a second copy
    # stream while step i computes, and the host waits for step i-1's result after launching
    # step i.
    copy_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)
    d_bufs = [d_buf, torch.empty_like(d_buf)]

    def views(buf):
        v = {}
        for k, t in parts.items():
            n = t.numel() * t.element_size()
            v[k] = buf[offs[k]:offs[k] + n].view(t.dtype).view(t.shape)
        return v

    d_ins = [d_in, views(d_bufs[1])]
    outs = [out, torch.empty_like(out)]
    h_outs = [h_out, torch.empty(out.shape, dtype=out.dtype).pin_memory()]
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]    # input copy of buffer j landed
    ev_used = [torch.cuda.Event(), torch.cuda.Event()]  # the step on buffer j has read it
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]   # the result of buffer j is on the host

    def pipe_step(i):
        j = i % 2
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(ev_used[j])
            d_bufs[j].copy_(h_buf, non_blocking=True)
            ev_in[j].record(copy_stream)
        stream.wait_event(ev_in[j])
        stream.wait_event(ev_out[j])  # outs[j]'s previous result (step i-2) has left the device
        kc, vc = pools[i % rot]
        dj = d_ins[j]
        if mapping is not None:
            pa.pa_copy_blocks(kc, vc, dj["mapping"])
        pa.pa_reshape_and_cache(dj["key"], dj["value"], kc, vc, dj["slots"])
        decode(dj["query"], kc, vc, dj["tables"], dj["lens"], o=outs[j])
        ev_used[j].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(ev_used[j])
            h_outs[j].copy_(outs[j], non_blocking=True)
            ev_out[j].record(d2h_stream)
        if i >= 1:
            ev_out[1 - j].synchronize()  # step i-1's result is on the host

    for i in range(min(args.warmup, 50)):
        pipe_step(i)
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    copy_stream.wait_event(p0)  # every copy of the timed region starts after p0
    d2h_stream.wait_event(p0)
    for i in range(args.steps):
        pipe_step(i)
    stream.wait_event(ev_out[(args.steps - 1) % 2])  # the region ends with the last result out
    p1.record(stream)
    ev_out[(args.steps - 1) % 2].synchronize()
    torch.cuda.synchronize()
    res["ms"] = p0.elapsed_time(p1)

    # where one eager end-to-end step's time goes: events between its operations, and the host
    # wall clock from the first call to the return of the synchronize
    n_b = max(20, min(args.steps, 200))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(n_b)]
    walls = []
    for i in range(n_b):
        t0 = time.perf_counter()
        e2e_step(i, evs[i])
        walls.append(time.perf_counter() - t0)
    torch.cuda.synchronize()
    seg = np.array([[ev[j].elapsed_time(ev[j + 1]) for j in range(4)] for ev in evs]) * 1e3
    gap = np.array([evs[i][0].elapsed_time(evs[i + 1][0]) for i in range(n_b - 1)]) * 1e3
    med = np.median(seg, 0)
    res["breakdown"] = {
        "h2d_copy_us": round(float(med[0]), 2), "write_us": round(float(med[1]), 2),
        "decode_us": round(float(med[2]), 2), "d2h_copy_us": round(float(med[3]), 2),
        "device_busy_us": round(float(med.sum()), 2),
        "step_to_step_us": round(float(np.median(gap)), 2),
        "host_wall_us": round(float(np.median(walls)) * 1e6, 2),
        "idle_between_steps_us": round(float(np.median(gap) - med.sum()), 2),
        "steps": n_b,
        "how": "medians over eager end-to-end steps with CUDA events between the operations "
               "(events serialise the write and the decode); step_to_step is the interval "
               "between the starts of consecutive steps, idle the part of it no operation of "
               "the step covers (host launch and synchronize)"}

    # The same end-to-end step with its four operations (input copy, pa_decode_step or its two
    # halves, output copy) captured in one CUDA graph per pool copy: one launch per step, still
    # a synchronize and a host read of the output every step.
    if args.decode_flags == pa.PA_DECODE_OVERLAP_PREVIOUS and world == 1 and not args.shared:
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
        for i in range(args.steps):
            graphs[i % rot].replay()
            stream.synchronize()
        g1.record(stream)
        torch.cuda.synchronize()
        res["graph_ms"] = g0.elapsed_time(g1)
        del graphs
    return res


def run_fp8(args, b, config, full: bool = True, probe: dict | None = None) -> dict:
    """The same decode step over an FP8 E4M3 cache: the pool is the workload's pool quantised
    (per-kv-head scales: largest magnitude of the head's rows / 240), and each step is one
    pa_decode_step_fp8 call (one kernel: the new tokens quantised into the caches, and the
    decode).  Timed like the 16-bit step: K steps with nothing between launches (`value`), then
    steps with events around each call (the roofline)."""
    import torch

    import paged_kv_cache_427_b200 as pa

    pa.load()
    dev = torch.device("cuda", 0)
    FP8 = torch.float8_e4m3fn

    kc16, vc16 = dev_tensor(b.key_cache, b.dtype, dev), dev_tensor(b.value_cache, b.dtype, dev)
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
    key, value = dev_tensor(b.key, b.dtype, dev), dev_tensor(b.value, b.dtype, dev)
    ks = (torch.cat([rows_k, key]).float().abs().amax(dim=(0, 2)) / 240.0).clamp_min(1e-8).contiguous()
    vs = (torch.cat([rows_v, value]).float().abs().amax(dim=(0, 2)) / 240.0).clamp_min(1e-8).contiguous()
    rot = pool_rotations(args, attended_bytes(b) // 2)
    pools = []
    for _ in range(rot):
        kc = torch.full(kc16.shape, 0x7f, dtype=torch.uint8, device=dev).view(FP8)
        vc = torch.full(vc16.shape, 0x7f, dtype=torch.uint8, device=dev).view(FP8)
        pa.pa_reshape_and_cache_fp8(rows_k, rows_v, kc, vc, su, ks, vs)
        pools.append((kc, vc))
    del kc16, vc16, rows_k, rows_v
    q = dev_tensor(b.query, b.dtype, dev)
    slots = dev_tensor(b.slot_mapping, None, dev)
    tables = dev_tensor(b.block_tables, None, dev)
    lens = dev_tensor(b.context_lens, None, dev)
    out = torch.empty(q.shape, dtype=q.dtype, device=dev)
    ws = torch.zeros(pa.pa_decode_workspace_bytes(b.num_seqs, b.num_heads, b.num_kv_heads,
                                                  b.head_dim, 0), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i, ev=None):
        kc, vc = pools[i % rot]
        if ev is not None:
            ev[0].record(stream)
        pa.pa_decode_step_fp8(key, value, kc, vc, slots, ks, vs, out, q, tables, lens, b.scale,
                              b.block_size, b.num_kv_heads, workspace=ws)
        if ev is not None:
            ev[1].record(stream)

    sampler = ClockSampler(None).start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    soak(step, args.soak if full else min(args.soak, 0.3))
    elapsed_ms = run_steps(step, args.steps, stream)
    dec_ms = run_launches(step, launch_count(args))
    timeline = None
    if full and args.timeline:
        workers = pa.pa_decode_default_workers(pa.PA_BF16, b.head_dim, b.block_size,
                                               b.num_heads // b.num_kv_heads)
        buf = torch.zeros(max(workers, 1) * 2 * pa.TIMELINE_WORDS, dtype=torch.int64, device=dev)
        pa.pa_set_decode_timeline(buf)
        recs = []
        try:
            for i in range(args.timeline):
                buf.zero_()
                step(i)
                torch.cuda.synchronize()
                recs.append(buf.cpu().numpy().copy())
        finally:
            pa.pa_set_decode_timeline(None)
        timeline = timeline_summary(recs, 16 * b.head_dim * 1 * 2)
        if args.timeline_out:
            np.save(args.timeline_out, np.stack(recs))
    clocks = sampler.stop()
    flags = pa.pa_get_device_error(clear=True)
    if flags:
        print(f"warning: device error word 0x{flags:x}", file=sys.stderr)
    dec = decode_bytes(b, ELT[b.dtype], unique=True, kv_elt=1)
    t_new = int((b.slot_mapping >= 0).sum())
    wbytes = t_new * b.num_kv_heads * b.head_dim * (ELT[b.dtype] + 1) * 2 + len(b.slot_mapping) * 8
    ms = elapsed_ms / args.steps
    value = (dec + wbytes) / (ms * 1e-3) / 1e9
    line = {"metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3 cache, bf16 query", "data": "synthetic",
            "config": dict(config, kv_dtype="fp8_e4m3", pool_rotations=rot,
                           kv_scales="per kv head: max |x| / 240"),
            "attended_tokens_per_s": round(b.attended_tokens / (ms * 1e-3), 1),
            "seq_steps_per_s": round(b.num_seqs / (ms * 1e-3), 1),
            "pct_of_8TBs": round(100 * value / NOMINAL_HBM_GBS, 2),
            "roofline": hbm_roofline(dec, dec_ms, "paged_decode_mma_kernel (fp8 e4m3 cache), fused "
                                     "step: the quantising cache write inside the same kernel",
                                     recorded_traffic(config["workload"] + ":fp8", "decode_fp8"),
                                     probe),
            "gpu_launches": args.steps, "clocks": clocks}
    if timeline:
        line["timeline"] = timeline
    if full and not args.no_cpu_baseline:
        kc8, vc8 = pools[0]
        line["cpu_baseline"] = cpu_baseline_fp8(
            b, kc8.view(torch.uint8).cpu().numpy(), vc8.view(torch.uint8).cpu().numpy(),
            ks.cpu().numpy(), vs.cpu().numpy(), args.cpu_seconds)
    return line


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


def run_prefill(args, b, config, full: bool = True) -> dict:
    """A chunked-prefill step: the new tokens' K/V written (pa_reshape_and_cache), then
    pa_prefill.  Timed like the decode step; the roofline is tensor-bound, against the measured
    bf16 dense GEMM rate (the burst figure: the kernel is timed alone per launch)."""
    import torch

    import paged_kv_cache_427_b200 as pa

    pa.load()
    dev = torch.device("cuda", 0)
    kc0, vc0 = dev_tensor(b.key_cache, b.dtype, dev), dev_tensor(b.value_cache, b.dtype, dev)
    rot = pool_rotations(args, attended_bytes(b))
    pools = [(kc0, vc0)] + [(kc0.clone(), vc0.clone()) for _ in range(rot - 1)]
    q = dev_tensor(b.query, b.dtype, dev)
    key, value = dev_tensor(b.key, b.dtype, dev), dev_tensor(b.value, b.dtype, dev)
    slots, tables = dev_tensor(b.slot_mapping, None, dev), dev_tensor(b.block_tables, None, dev)
    lens, qs = dev_tensor(b.context_lens, None, dev), dev_tensor(b.query_start, None, dev)
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
    soak(step, args.soak if full else min(args.soak, 0.3), per_round=50)
    elapsed_ms = run_steps(step, args.steps, stream)
    k_ms = run_launches(step, launch_count(args))
    clocks = sampler.stop()
    flags = pa.pa_get_device_error(clear=True)
    if flags:
        print(f"warning: device error word 0x{flags:x}", file=sys.stderr)
    flops = prefill_flops(b)
    ms = elapsed_ms / args.steps
    peak, src = bf16_peak()
    st = launch_stats(k_ms)
    tflops = flops / (st["mean_launch_us"] * 1e-6) / 1e12
    new_tokens = int(b.query_start[-1])
    traffic = recorded_traffic(config["workload"], "prefill")
    line = {"metric": PREFILL_METRIC, "value": round(flops / (ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": b.dtype, "data": "synthetic",
            "config": dict(config, new_tokens=new_tokens, pool_rotations=rot,
                           query_lens=[int(x) for x in np.diff(b.query_start)]),
            "new_tokens_per_s": round(new_tokens / (ms * 1e-3), 1),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "traffic": traffic,
                         "kernel": "paged_prefill_tc_kernel (tcgen05 + TMEM + TMA)",
                         "peak_source": src, "algorithmic_flops_per_launch": flops, **st},
            "gpu_launches": args.steps, "clocks": clocks}
    if full and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_prefill(b, args.cpu_seconds)
    return line


# The other workloads of the default run, after the Llama-3-8B-shaped headline: the long
# mixed batch (its own >= 60 % bar), the block-size sweep, the shared prefix, the FP8 cache on
# the headline's batch and the chunked prefill.
CONFIG_RUNS = (("long_mixed", "decode"), ("short_chat_bs8", "decode"), ("short_chat_bs16", "decode"),
               ("short_chat_bs32", "decode"), ("shared_prefix", "shared"),
               ("shared_prefix", "decode"), ("llama3_8b_decode", "fp8"),
               ("chunked_prefill", "prefill"))


def run_configs(args, probe) -> dict:
    """One compact record per workload of CONFIG_RUNS, each measured like the headline (K
    steps, then per-launch events), without the end-to-end, graph and CPU legs."""
    import torch

    keep = ("metric", "value", "unit", "ms_per_step", "pct_of_8TBs", "pct_of_read_probe",
            "attended_tokens_per_s", "seq_steps_per_s", "new_tokens_per_s", "logical_GBps",
            "roofline", "clocks", "dtype", "decode_call")
    res = {}
    for name, kind in CONFIG_RUNS:
        b = make_batch(name)
        cfg = workload_config(args, b, name)
        if kind == "fp8":
            line = run_fp8(args, b, cfg, full=False, probe=probe)
            key = name + ":fp8"
        elif kind == "prefill":
            line = run_prefill(args, b, cfg, full=False)
            key = name
        elif kind == "shared":
            line = run_decode(args, b, cfg, full=False, probe=probe, shared=True)
            key = name
        else:
            line = run_decode(args, b, cfg, full=False, probe=probe)
            key = name + (":pa_decode" if name == "shared_prefix" else "")
        rec = {k: line[k] for k in keep if k in line}
        rec["config"] = {k: v for k, v in line["config"].items()
                         if k in ("num_seqs", "block_size", "attended_tokens", "kv_dtype",
                                  "new_tokens", "num_blocks")}
        res[key] = rec
        del b
        torch.cuda.empty_cache()
    return res


def workload_config(args, b, name: str) -> dict:
    return {"workload": name, "num_seqs": b.num_seqs, "num_heads": b.num_heads,
            "num_kv_heads": b.num_kv_heads, "head_dim": b.head_dim, "block_size": b.block_size,
            "kv_dtype": b.dtype, "attended_tokens": b.attended_tokens,
            "num_blocks": b.num_blocks, "max_blocks_per_seq": b.max_blocks,
            "seed": b.meta.get("seed"),
            "l2": "inputs larger than L2: steps rotate over copies of the KV pool",
            "pool_rotations": args.rotations or "auto",
            "decode_flags": args.decode_flags}


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
    ap.add_argument("--workload", default=None,
                    help="llama3_8b_decode (default) | short_chat_bs{8,16,32} | shared_prefix | "
                         "long_mixed | tiny_fp32 | chunked_prefill (pa_prefill)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-flags", type=int, default=4,
                    help="pa_decode_ex flags: 4 = start while the cache write runs (default), "
                         "2 = CUDA-core kernel, 1 = separate merge kernel, 0 = plain pa_decode")
    ap.add_argument("--rotations", type=int, default=0, help="copies of the KV pool (0 = enough to defeat L2)")
    ap.add_argument("--soak", type=float, default=1.0, help="seconds of untimed load for the clock sampler")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="the default run: skip the other workloads (the `configs` key)")
    ap.add_argument("--no-probe", action="store_true", help="skip the read-only HBM probe")
    ap.add_argument("--timeline", type=int, default=0, metavar="N",
                    help="record N decode launches with pa_set_decode_timeline and add a summary")
    ap.add_argument("--timeline-out", default=None, help="save the raw timeline records (.npy)")
    ap.add_argument("--shared", action="store_true",
                    help="decode the workload with pa_decode_shared_prefix over its groups")
    ap.add_argument("--kv", default="native", choices=["native", "fp8"],
                    help="fp8: the same step over an FP8 E4M3 cache (pa_decode_fp8)")
    ap.add_argument("--swap", action="store_true",
                    help="measure block swap (pa_swap_blocks) of the workload's blocks instead")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    default_run = args.workload is None
    workload = args.workload or "llama3_8b_decode"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        args.gpus = world if world > 1 else args.gpus
    b = make_batch(workload)
    config = workload_config(args, b, workload)
    config["parallelism"] = f"replicas x{world}" if world > 1 else "single GPU"

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
            print(json.dumps(run_fp8(args, b, config)), flush=True)
        return
    if b.query_start is not None:
        if rank == 0:
            print(json.dumps(run_prefill(args, b, config)), flush=True)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        probe = None
        if world == 1 and not args.no_probe:
            probe = read_probe(torch.device("cuda", local_rank))
        line = run_decode(args, b, config, rank, world, local_rank, full=True, probe=probe,
                          shared=args.shared)
        if line is not None:
            if probe:
                line["hbm_read_probe"] = probe
            if default_run and world == 1 and not args.no_configs:
                del b
                torch.cuda.empty_cache()
                line["configs"] = run_configs(args, probe)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
