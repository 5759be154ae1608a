"""Helpers for the GPU parity tests: move a seeded batch to the device, run the library's step
through the C ABI, and compare against the CPU oracle's step on host copies of the same bytes.

Tolerances (fixed before any kernel ran; the bf16-output bound restated from the kernels'
arithmetic as below):
  * cache writes and block copies: bit-exact;
  * fp32 caches with fp32 output: max abs error <= 1e-5 and relative L2 error <= 1e-5;
  * bf16 / fp16 caches with fp32 output: max abs error <= 5e-3 and relative L2 <= 1e-3;
  * bf16 output: every element within one bf16 ulp of the fp64 result o plus
    2^-16 * max_{t<L} |V_t - o| (the error the fp32 result may carry before its one rounding:
    each softmax weight is kept to 2^-18 relative by the hi + lo split of P, 2^-22 by exp2,
    and the fp32 logit and sums add a few 2^-24 per step; a relative error e on the weights
    moves o by at most e * max_t |V_t - o|; 2^-16 allows four times the split's share), and at
    least 99% of the elements equal to o rounded to nearest-even bf16 (an element whose exact
    value lies within that error of a rounding midpoint may round either way).
The achieved figures of every comparison are collected in RESULTS and printed at the end of
the pytest run (tests/conftest.py).
"""
from __future__ import annotations

import numpy as np
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W

TOL = {"f32": (1e-5, 1e-5), "bf16": (5e-3, 1e-3), "f16": (5e-3, 1e-3)}
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pa.load()


def to_torch(a: np.ndarray, dtype: str | None = None, device="cuda") -> torch.Tensor:
    """Host array -> device tensor with the same bytes (bf16 stored as uint16 patterns)."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device)


def to_host(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


class DeviceBatch:
    """Device copies of a batch's inputs."""

    def __init__(self, b: W.PagedBatch, device="cuda"):
        self.b = b
        dt = b.dtype
        self.query = to_torch(b.query, dt, device)
        self.key_cache = to_torch(b.key_cache, dt, device)
        self.value_cache = to_torch(b.value_cache, dt, device)
        self.key = to_torch(b.key, dt, device)
        self.value = to_torch(b.value, dt, device)
        self.slot_mapping = to_torch(b.slot_mapping, None, device)
        self.block_tables = to_torch(b.block_tables, None, device)
        self.context_lens = to_torch(b.context_lens, None, device)
        self.block_mapping = (to_torch(b.block_mapping, None, device)
                              if b.block_mapping is not None and len(b.block_mapping) else None)

    def write(self):
        if self.block_mapping is not None:
            pa.pa_copy_blocks(self.key_cache, self.value_cache, self.block_mapping)
        pa.pa_reshape_and_cache(self.key, self.value, self.key_cache, self.value_cache,
                                self.slot_mapping)

    def decode(self, out_dtype: str, num_workers: int | None = None, flags: int = 0,
               workspace: torch.Tensor | None = None, query=None, out=None) -> torch.Tensor:
        b = self.b
        q = self.query if query is None else query
        if out is None:
            out = torch.empty(q.shape, dtype=TORCH_DTYPE[out_dtype], device=q.device)
        if num_workers is None and not flags and workspace is None:
            # pa_decode: library-owned workspace, default kernel and worker count
            pa.pa_decode(out, q, self.key_cache, self.value_cache, self.block_tables,
                         self.context_lens, b.scale, b.block_size, b.num_kv_heads)
        else:
            if workspace is None:
                n = pa.pa_decode_workspace_bytes(q.shape[0], q.shape[1], b.num_kv_heads,
                                                 b.head_dim, num_workers or 0)
                workspace = torch.zeros(n, dtype=torch.uint8, device=q.device)
            pa.pa_decode_ex(out, q, self.key_cache, self.value_cache, self.block_tables,
                            self.context_lens, b.scale, b.block_size, b.num_kv_heads,
                            num_workers=num_workers or 0, flags=flags, workspace=workspace)
        return out


def oracle_step(orc, b: W.PagedBatch, seqs=None):
    """The oracle's copies, writes and decode on host copies of the pool.  With `seqs`, decode
    only those sequences.  Returns (out float64, key_cache, value_cache)."""
    kc = b.key_cache.copy()
    vc = b.value_cache.copy()
    if b.block_mapping is not None and len(b.block_mapping):
        assert orc.copy_blocks(kc, vc, b.block_mapping, b.dtype) == 0
    assert orc.reshape_and_cache(b.key, b.value, kc, vc, b.slot_mapping, b.dtype) == 0
    if seqs is None:
        out = orc.decode(b.query, kc, vc, b.block_tables, b.context_lens, b.scale, b.dtype)
    else:
        sub = W.sub_batch(b, seqs)
        out = orc.decode(sub["query"], kc, vc, sub["block_tables"], sub["context_lens"],
                         b.scale, b.dtype)
    return out, kc, vc


def errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    abs_err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel_l2 = float(np.linalg.norm(got - ref) / denom) if denom > 0 else abs_err
    return abs_err, rel_l2


RESULTS: list = []  # (what, kind, figures) of every comparison, printed after the run


def assert_close(got, ref, dtype: str, what: str = ""):
    atol, rtol = TOL[dtype]
    a, r = errors(got, ref)
    RESULTS.append((what, "fp32 out", f"max abs {a:.2e} (<= {atol}), rel L2 {r:.2e} (<= {rtol})"))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert a <= atol and r <= rtol, f"{what}: max abs {a:.3e} (<= {atol}), rel L2 {r:.3e} (<= {rtol})"
    return a, r


_FP8_VALUES = None


def _fp8_values() -> np.ndarray:
    """float64 value of each E4M3 code (torch's decoder; NaN codes decode to NaN)."""
    global _FP8_VALUES
    if _FP8_VALUES is None:
        _FP8_VALUES = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    return _FP8_VALUES


def value_spread(vc: np.ndarray, dtype: str, block_tables, context_lens, ref: np.ndarray,
                 block_size: int, row_seq=None, v_scale=None) -> np.ndarray:
    """max over the context (t < L) of |V_t[d] - o[d]| for every output element, ref's shape.
    vc: the value cache after the step's write, as stored (dtype "bf16", "f16", "f32" or "fp8"
    codes with per-kv-head v_scale); row_seq[r]: the sequence of output row r (default: row s is
    sequence s).  For a prefill row the context up to its position is part of t < L, so the
    spread over t < L bounds it."""
    rows_n, hq, d = ref.shape
    hkv = vc.shape[1]
    g = hq // hkv
    row_seq = np.arange(rows_n) if row_seq is None else np.asarray(row_seq)
    out = np.zeros(ref.shape, dtype=np.float64)
    for s in np.unique(row_seq):
        L = int(context_lens[s])
        rows = np.nonzero(row_seq == s)[0]
        if L <= 0 or rows.size == 0:
            continue
        t = np.arange(L)
        v = vc[block_tables[s, t // block_size], :, t % block_size, :]  # [L, Hkv, D]
        if dtype == "fp8":
            v = _fp8_values()[v] * np.asarray(v_scale, np.float64)[None, :, None]
        else:
            v = W.decode_to_f64(v, dtype)
        vmax = np.repeat(v.max(0), g, axis=0)  # [Hq, D]
        vmin = np.repeat(v.min(0), g, axis=0)
        o = ref[rows]
        out[rows] = np.maximum(np.abs(vmax - o), np.abs(vmin - o))
    return out


def assert_bf16_output(got_bits: np.ndarray, ref: np.ndarray, what: str, spread: np.ndarray):
    """bf16 output against the fp64 result o: |got - o| <= ulp(o) + 2^-16 * spread element by
    element (spread from value_spread), and >= 99% of the elements exactly RNE(o)."""
    got = W.bf16_bits_to_f32(got_bits).astype(np.float64)
    rne = W.f32_to_bf16_bits(ref.astype(np.float32))
    mag = np.maximum(np.abs(ref), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    bound = ulp + 2.0 ** -16 * spread
    err = np.abs(got - ref)
    worst = float(np.max(err / bound)) if err.size else 0.0
    same = float(np.mean(got_bits == rne)) if err.size else 1.0
    RESULTS.append((what, "bf16 out", f"{100 * same:.3f}% equal RNE(oracle) (>= 99%), largest "
                                      f"error {worst:.3f} of its bound (<= 1)"))
    assert np.all(err <= bound), f"{what}: bf16 output error {worst:.3f} times its bound"
    assert same >= 0.99, f"{what}: only {same:.4f} of bf16 outputs equal RNE(oracle)"
    return same


def assert_no_device_error():
    flags = pa.pa_get_device_error(clear=True)
    assert flags == 0, f"device error word 0x{flags:x}"


def assert_rounded_from(got_bits: np.ndarray, f32_out: np.ndarray, what: str = ""):
    """A bf16 output equals the nearest-even rounding of the same launch configuration's fp32
    output (the kernel accumulates identically and rounds once at the end)."""
    assert np.array_equal(got_bits, W.f32_to_bf16_bits(f32_out)), f"{what}: bf16 != RNE(fp32 out)"
