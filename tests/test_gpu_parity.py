"""Parity of the CUDA path (through the C ABI) with the CPU oracle on the same seeded inputs.

Cache writes and block copies must match bit for bit; attention must meet the tolerances in
tests/gpu_helpers.py.  Every test compares every output row with the oracle, the full-size
workloads included.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import (DeviceBatch, assert_bf16_output, assert_close,
                               assert_no_device_error, assert_rounded_from, oracle_step,
                               require_gpu, to_host, value_spread)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    pa.pa_get_device_error(clear=True)
    yield


def _spread(b, vc, ref):
    return value_spread(vc, b.dtype, b.block_tables, b.context_lens, ref, b.block_size)


def _check_caches(db, kc, vc, dtype):
    assert np.array_equal(to_host(db.key_cache, dtype).view(np.uint8), kc.view(np.uint8)), "key cache"
    assert np.array_equal(to_host(db.value_cache, dtype).view(np.uint8), vc.view(np.uint8)), "value cache"


# ------------------------------------------------------------------------------------------
# the five workloads
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("workers", [None, 1, 2, 3, 5, 64])
def test_tiny_fp32(oracle, workers):
    b = W.tiny_fp32()
    db = DeviceBatch(b)
    db.write()
    ref, kc, vc = oracle_step(oracle, b)
    _check_caches(db, kc, vc, "f32")
    out = db.decode("f32", num_workers=workers)
    assert_close(to_host(out, "f32"), ref, "f32", f"tiny fp32 W={workers}")
    assert_no_device_error()


@pytest.fixture(scope="module")
def llama_small(oracle):
    b = W.llama3_8b_decode(num_seqs=12, min_len=1, max_len=300)
    ref, kc, vc = oracle_step(oracle, b)
    return b, ref, kc, vc, _spread(b, vc, ref)


@pytest.mark.parametrize("workers,flags", [(None, 0), (1, 0), (7, 0), (33, 0), (512, 0),
                                           (5000, 0), (7, 1), (512, 1), (None, 1),
                                           (None, 2), (1, 2), (33, 2), (512, 3),
                                           (None, 4), (7, 4), (512, 5), (None, 6)])
def test_llama_small_workers(llama_small, workers, flags):
    b, ref, kc, vc, spread = llama_small
    db = DeviceBatch(b)
    db.write()
    _check_caches(db, kc, vc, "bf16")
    out = to_host(db.decode("f32", num_workers=workers, flags=flags), "f32")
    assert_close(out, ref, "bf16", f"W={workers} flags={flags}")
    outb = to_host(db.decode("bf16", num_workers=workers, flags=flags), "bf16")
    assert_bf16_output(outb, ref, f"bf16 out W={workers} flags={flags}", spread)
    assert_rounded_from(outb, out, f"bf16 out W={workers}")
    assert_no_device_error()


def test_llama_full_size(oracle):
    """Full Llama-3-8B-shaped step in the launch configuration the benchmark times; the
    oracle decodes every one of its 64 sequences."""
    b = W.llama3_8b_decode()
    db = DeviceBatch(b)
    db.write()
    # as the benchmark times it: bf16 out, decode overlapping the cache write just before it
    outb = db.decode("bf16", flags=pa.PA_DECODE_OVERLAP_PREVIOUS)
    out = db.decode("f32")
    torch.cuda.synchronize()
    ref, kc, vc = oracle_step(oracle, b)
    _check_caches(db, kc, vc, "bf16")
    assert_close(to_host(out, "f32"), ref, "bf16", "llama full (every sequence)")
    assert_bf16_output(to_host(outb, "bf16"), ref, "llama full bf16 (every sequence)",
                       _spread(b, vc, ref))
    assert_no_device_error()


def test_short_chat_block_sizes(oracle):
    outs = {}
    ref0 = None
    for bs in (8, 16, 32):
        b = W.short_chat(bs)
        db = DeviceBatch(b)
        db.write()
        ref, kc, vc = oracle_step(oracle, b)
        _check_caches(db, kc, vc, "bf16")
        out = to_host(db.decode("f32"), "f32")
        assert_close(out, ref, "bf16", f"short chat bs={bs}")
        outb = to_host(db.decode("bf16"), "bf16")
        assert_bf16_output(outb, ref, f"short chat bf16 bs={bs}", _spread(b, vc, ref))
        if ref0 is None:
            ref0 = ref
        assert np.array_equal(ref, ref0), "oracle differs across block sizes"
        outs[bs] = out
    for bs in (16, 32):
        assert_close(outs[bs], outs[8], "bf16", f"bs {bs} vs bs 8")
    assert_no_device_error()


def test_shared_prefix(oracle):
    b = W.shared_prefix()
    db = DeviceBatch(b)
    db.write()
    ref, kc, vc = oracle_step(oracle, b)
    _check_caches(db, kc, vc, "bf16")
    assert_close(to_host(db.decode("f32"), "f32"), ref, "bf16", "shared prefix")
    assert_bf16_output(to_host(db.decode("bf16"), "bf16"), ref, "shared prefix bf16",
                       _spread(b, vc, ref))
    assert_no_device_error()


def test_long_mixed_full_size(oracle):
    """The long mixed batch at full size (16 contexts of 8k-32k tokens split over many warps,
    240 short ones); the oracle decodes all 256 sequences."""
    b = W.long_mixed()
    db = DeviceBatch(b)
    db.write()
    out = db.decode("f32")
    outb = db.decode("bf16", flags=pa.PA_DECODE_OVERLAP_PREVIOUS)
    outs = db.decode("f32", flags=pa.PA_DECODE_SEPARATE_REDUCE)
    outc = db.decode("f32", flags=pa.PA_DECODE_CUDA_CORES)
    torch.cuda.synchronize()
    ref, kc, vc = oracle_step(oracle, b)
    _check_caches(db, kc, vc, "bf16")
    assert_close(to_host(out, "f32"), ref, "bf16", "long mixed (every sequence)")
    assert_close(to_host(outs, "f32"), ref, "bf16", "long mixed separate reduce")
    assert_close(to_host(outc, "f32"), ref, "bf16", "long mixed CUDA-core kernel")
    assert_bf16_output(to_host(outb, "bf16"), ref, "long mixed bf16 (every sequence)",
                       _spread(b, vc, ref))
    assert_no_device_error()


# ------------------------------------------------------------------------------------------
# invariants, variants and edge cases
# ------------------------------------------------------------------------------------------

def _gpu_out(b, out_dtype="f32", **kw):
    db = DeviceBatch(b)
    db.write()
    return to_host(db.decode(out_dtype, **kw), out_dtype)


def test_placement_and_poison_invariance():
    """Same logical values: other permutation, zero instead of NaN in unread slots, garbage in
    unread block-table entries -> bit-identical output (the kernel walks logical order)."""
    base = dict(num_seqs=10, min_len=1, max_len=200)
    for flags in (0, pa.PA_DECODE_CUDA_CORES):
        ref = _gpu_out(W.llama3_8b_decode(**base), num_workers=97, flags=flags)
        b = W.llama3_8b_decode(**base, fill="zero")
        assert np.array_equal(_gpu_out(b, num_workers=97, flags=flags), ref)
        b = W.llama3_8b_decode(**base)
        b.block_tables = np.where(b.block_tables < 0, np.int32(2 ** 30), b.block_tables)
        assert np.array_equal(_gpu_out(b, num_workers=97, flags=flags), ref)
        b = W.build_batch("perm", W.llama3_8b_decode(**base).context_lens, num_heads=32,
                          num_kv_heads=8, head_dim=128, block_size=16, dtype="bf16",
                          seed=W.BASE_SEED + 2, perm_salt=5, max_blocks=13)
        assert np.array_equal(_gpu_out(b, num_workers=97, flags=flags), ref)
    assert_no_device_error()


def test_repeated_calls_are_identical():
    """The merge counters reset themselves: back-to-back calls give identical bits."""
    b = W.llama3_8b_decode(num_seqs=16, min_len=1, max_len=2048)
    db = DeviceBatch(b)
    db.write()
    first = to_host(db.decode("f32"), "f32")
    for _ in range(3):
        assert np.array_equal(to_host(db.decode("f32"), "f32"), first)
    n = pa.pa_decode_workspace_bytes(16, 32, 8, 128, 300)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    a = to_host(db.decode("f32", num_workers=300, workspace=ws), "f32")
    for _ in range(3):
        assert np.array_equal(to_host(db.decode("f32", num_workers=300, workspace=ws), "f32"), a)
    assert_no_device_error()


@pytest.mark.parametrize("dtype,D,bs,hq,hkv", [
    ("bf16", 64, 8, 8, 8), ("bf16", 64, 32, 16, 8), ("bf16", 128, 8, 16, 2),
    ("bf16", 128, 32, 32, 4), ("f16", 128, 16, 32, 8), ("f16", 64, 16, 8, 1),
    ("f32", 128, 16, 16, 2), ("f32", 128, 32, 8, 8), ("f32", 64, 8, 32, 4),
])
def test_configuration_coverage(oracle, dtype, D, bs, hq, hkv):
    rng = np.random.default_rng([D, bs, hq])
    lens = rng.integers(1, 700, size=6).astype(np.int32)
    lens[0] = 1
    lens[1] = bs * 3
    b = W.build_batch("cov", lens, num_heads=hq, num_kv_heads=hkv, head_dim=D, block_size=bs,
                      dtype=dtype, seed=W.BASE_SEED + 900 + D + bs)
    ref, kc, vc = oracle_step(oracle, b)
    variants = [(None, 0), (5, 0)] + ([(None, pa.PA_DECODE_CUDA_CORES), (5, pa.PA_DECODE_CUDA_CORES)]
                                      if dtype != "f32" else [])
    for workers, flags in variants:
        db = DeviceBatch(b)
        db.write()
        _check_caches(db, kc, vc, dtype)
        what = f"{dtype} D{D} bs{bs} G{hq // hkv} W={workers} flags={flags}"
        assert_close(to_host(db.decode("f32", num_workers=workers, flags=flags), "f32"), ref,
                     dtype, what)
        if dtype != "f32":
            got = to_host(db.decode(dtype, num_workers=workers, flags=flags), dtype)
            if dtype == "bf16":
                assert_bf16_output(got, ref, "bf16 out " + what, _spread(b, vc, ref))
            else:
                assert_close(got.astype(np.float64), ref, dtype, "fp16 out " + what)
    assert_no_device_error()


def test_empty_and_extreme_contexts(oracle):
    lens = np.array([0, 5, 0, 1, 16 * 13, 0], np.int32)
    b = W.build_batch("edge", lens, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                      dtype="bf16", seed=W.BASE_SEED + 950, max_blocks=13)
    ref, _, _ = oracle_step(oracle, b)
    for workers in (None, 1, 4, 50):
        for flags in (0, pa.PA_DECODE_CUDA_CORES):
            got = _gpu_out(b, num_workers=workers, flags=flags)
            assert np.all(got[[0, 2, 5]] == 0)
            assert_close(got, ref, "bf16", f"edge W={workers} flags={flags}")
    b0 = W.build_batch("allzero", [0, 0, 0], num_heads=8, num_kv_heads=2, head_dim=64,
                       block_size=8, dtype="bf16", seed=1, max_blocks=2)
    assert np.all(_gpu_out(b0) == 0)
    assert_no_device_error()


def test_single_very_long_sequence(oracle):
    """One sequence of 32768 tokens split over every warp of the device."""
    b = W.build_batch("long1", [32768], num_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=16, dtype="bf16", seed=W.BASE_SEED + 960)
    ref, _, _ = oracle_step(oracle, b)
    for flags in (0, pa.PA_DECODE_SEPARATE_REDUCE, pa.PA_DECODE_CUDA_CORES):
        assert_close(_gpu_out(b, flags=flags), ref, "bf16", f"32k tokens flags={flags}")
    assert_no_device_error()


def test_strided_query_and_out(oracle):
    b = W.llama3_8b_decode(num_seqs=5, min_len=1, max_len=300)
    ref, _, _ = oracle_step(oracle, b)
    db = DeviceBatch(b)
    db.write()
    big = torch.zeros((5, 32, 256), dtype=torch.bfloat16, device="cuda")
    big[:, :, 64:192] = db.query
    q = big[:, :, 64:192]                          # heads not contiguous: one copy per head
    for flags in (0, pa.PA_DECODE_CUDA_CORES):
        outbig = torch.zeros((5, 40, 128), dtype=torch.float32, device="cuda")
        out = outbig[:, 4:36, :]
        db.decode("f32", query=q, out=out, flags=flags)
        assert_close(to_host(out, "f32"), ref, "bf16", f"strided flags={flags}")
        assert torch.all(outbig[:, :4] == 0) and torch.all(outbig[:, 36:] == 0)
    assert_no_device_error()


def test_write_side_padding_and_bad_slots():
    b = W.tiny_fp32()
    db = DeviceBatch(b)
    slots = db.slot_mapping.clone()
    slots[1] = -1
    slots[2] = b.num_blocks * b.block_size
    before = to_host(db.key_cache, "f32").copy()
    pa.pa_reshape_and_cache(db.key, db.value, db.key_cache, db.value_cache, slots)
    flags = pa.pa_get_device_error(clear=True)
    assert flags == pa.PA_DEVERR_SLOT
    after = to_host(db.key_cache, "f32")
    expect = before.copy()
    for s in (0, 3):
        blk, off = divmod(int(b.slot_mapping[s]), b.block_size)
        expect[blk, :, off] = b.key[s]
    assert np.array_equal(after.view(np.uint8), expect.view(np.uint8))


def test_copy_blocks_bit_exact_and_bad_pairs(oracle):
    b = W.llama3_8b_decode(num_seqs=4, min_len=100, max_len=300, fill="zero")
    rng = np.random.default_rng(11)
    b.key_cache = W.encode(rng.standard_normal(b.key_cache.shape, dtype=np.float32), "bf16")
    b.value_cache = W.encode(rng.standard_normal(b.value_cache.shape, dtype=np.float32), "bf16")
    pairs = np.array([[3, 60], [7, 5], [3, 9]], np.int64)
    db = DeviceBatch(b)
    pa.pa_copy_blocks(db.key_cache, db.value_cache, torch.from_numpy(pairs).cuda())
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    assert oracle.copy_blocks(kc, vc, pairs, "bf16") == 0
    _check_caches(db, kc, vc, "bf16")
    assert_no_device_error()
    bad = torch.tensor([[0, b.num_blocks], [-2, 4], [1, 2]], dtype=torch.int64, device="cuda")
    pa.pa_copy_blocks(db.key_cache, db.value_cache, bad)
    assert pa.pa_get_device_error(clear=True) == pa.PA_DEVERR_COPY_PAIR
    assert oracle.copy_blocks(kc, vc, bad.cpu().numpy(), "bf16") == 2
    _check_caches(db, kc, vc, "bf16")


def test_bad_block_ids_and_lengths_are_flagged():
    b = W.llama3_8b_decode(num_seqs=4, min_len=40, max_len=100)
    b.block_tables = b.block_tables.copy()
    b.block_tables[2, 1] = b.num_blocks + 5      # inside the context of sequence 2
    out = _gpu_out(b)
    assert np.all(np.isfinite(out[[0, 1, 3]]))
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_BLOCK_ID
    b = W.llama3_8b_decode(num_seqs=4, min_len=40, max_len=100)
    b.context_lens = b.context_lens.copy()
    b.context_lens[1] = b.max_blocks * b.block_size + 7
    b.context_lens[3] = -3
    b.slot_mapping = b.slot_mapping.copy()
    b.slot_mapping[[1, 3]] = -1
    out = _gpu_out(b)
    assert np.all(out[3] == 0)
    # the clamped context of sequence 1 also reaches block-table entries past its blocks
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_CONTEXT_LEN


def test_decode_and_decode_ex_agree():
    b = W.llama3_8b_decode(num_seqs=20, min_len=1, max_len=2048)
    db = DeviceBatch(b)
    db.write()
    w = pa.pa_decode_default_workers(pa.PA_BF16, 128, 16, 4)
    assert w > 0
    a = to_host(db.decode("f32"), "f32")
    c = to_host(db.decode("f32", num_workers=w), "f32")
    assert np.array_equal(a, c)
    assert_no_device_error()
