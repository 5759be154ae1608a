"""Helpers for the GPU parity tests: move a seeded batch to the device, run the library's step
through the C ABI, and compare against the CPU oracle's step on host copies of the same bytes.

Tolerances (fixed before any kernel ran):
  * cache writes and block copies: bit-exact;
  * fp32 caches with fp32 output: max abs error <= 1e-5 and relative L2 error <= 1e-5;
  * bf16 / fp16 caches with fp32 output: max abs error <= 5e-3 and relative L2 <= 1e-3;
  * bf16 output: each element within one bf16 ulp of the fp64 result plus 1e-5 (the fp32
    accumulation error of outputs near zero exceeds their ulp), and at least 99% of the
    elements equal to that result rounded to nearest-even bf16.
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


def assert_close(got, ref, dtype: str, what: str = ""):
    atol, rtol = TOL[dtype]
    a, r = errors(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert a <= atol and r <= rtol, f"{what}: max abs {a:.3e} (<= {atol}), rel L2 {r:.3e} (<= {rtol})"
    return a, r


def assert_bf16_output(got_bits: np.ndarray, ref: np.ndarray, what: str = ""):
    """bf16 output against the fp64 result: within one ulp + 1e-5, >= 99% exactly RNE(ref)."""
    got = W.bf16_bits_to_f32(got_bits).astype(np.float64)
    rne = W.f32_to_bf16_bits(ref.astype(np.float32))
    mag = np.maximum(np.abs(ref), 2.0 ** -126)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    worst = float(np.max((np.abs(got - ref) - 1e-5) / ulp))
    assert np.all(np.abs(got - ref) <= ulp + 1e-5), f"{what}: bf16 output off by {worst:.2f} ulp + 1e-5"
    same = float(np.mean(got_bits == rne))
    assert same >= 0.99, f"{what}: only {same:.4f} of bf16 outputs equal RNE(oracle)"
    return same


def assert_no_device_error():
    flags = pa.pa_get_device_error(clear=True)
    assert flags == 0, f"device error word 0x{flags:x}"


def assert_rounded_from(got_bits: np.ndarray, f32_out: np.ndarray, what: str = ""):
    """A bf16 output equals the nearest-even rounding of the same launch configuration's fp32
    output (the kernel accumulates identically and rounds once at the end)."""
    assert np.array_equal(got_bits, W.f32_to_bf16_bits(f32_out)), f"{what}: bf16 != RNE(fp32 out)"
