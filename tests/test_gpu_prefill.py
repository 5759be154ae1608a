"""pa_prefill: causal attention of each sequence's new tokens over the paged cache, compared
with the oracle (fp32 out within the 16-bit tolerance, 16-bit out against the rounding of the
fp64 result) on a mixed continuously batched step (whole prompts, prompt chunks on top of a
prefix, single decode tokens, a sequence with no new token), for every built configuration, on
the full-size chunked-prefill workload (every sequence), and on its error cases."""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import (TORCH_DTYPE, assert_bf16_output, assert_close, value_spread,
                               assert_no_device_error, require_gpu, to_host, to_torch)

pytestmark = pytest.mark.gpu


class PrefillStep:
    def __init__(self, b):
        self.b = b
        dt = b.dtype
        self.query = to_torch(b.query, dt)
        self.key_cache = to_torch(b.key_cache, dt)
        self.value_cache = to_torch(b.value_cache, dt)
        self.key, self.value = to_torch(b.key, dt), to_torch(b.value, dt)
        self.slots = to_torch(b.slot_mapping)
        self.tables = to_torch(b.block_tables)
        self.lens = to_torch(b.context_lens)
        self.qs = to_torch(b.query_start)
        pa.pa_reshape_and_cache(self.key, self.value, self.key_cache, self.value_cache, self.slots)

    def run(self, out_dtype):
        b = self.b
        out = torch.full(self.query.shape, float("nan"), dtype=TORCH_DTYPE[out_dtype], device="cuda")
        pa.pa_prefill(out, self.query, self.key_cache, self.value_cache, self.tables, self.lens,
                      self.qs, b.scale, b.block_size, b.num_kv_heads)
        return to_host(out, out_dtype)


def _spread(b, vc, ref):
    """value_spread for prefill rows: row r belongs to the sequence whose new tokens hold it."""
    row_seq = np.repeat(np.arange(b.num_seqs), np.diff(b.query_start))
    return value_spread(vc, b.dtype, b.block_tables, b.context_lens, ref, b.block_size,
                        row_seq=row_seq)


def _oracle(orc, b):
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    assert orc.reshape_and_cache(b.key, b.value, kc, vc, b.slot_mapping, b.dtype) == 0
    ref = orc.prefill(b.query, kc, vc, b.block_tables, b.context_lens, b.query_start, b.scale, b.dtype)
    return ref, kc, vc


def test_prefill_mixed_batch(oracle):
    require_gpu()
    b = W.build_prefill_batch("pf", [300, 77, 16, 1, 640, 33, 200, 95],
                              [300, 13, 16, 1, 128, 0, 1, 95], num_heads=32, num_kv_heads=8,
                              head_dim=128, block_size=16, dtype="bf16", seed=W.BASE_SEED + 740)
    ref, kc, vc = _oracle(oracle, b)
    st = PrefillStep(b)
    assert np.array_equal(to_host(st.key_cache, "bf16"), kc)
    assert np.array_equal(to_host(st.value_cache, "bf16"), vc)
    assert_close(st.run("f32"), ref, "bf16", "prefill mixed batch")
    assert_bf16_output(st.run("bf16"), ref, "prefill bf16 out", _spread(b, vc, ref))
    assert_no_device_error()


@pytest.mark.parametrize("dtype,D,bs,hq,hkv", [
    ("bf16", 64, 8, 8, 8), ("bf16", 64, 32, 16, 8), ("bf16", 128, 8, 16, 2),
    ("bf16", 128, 32, 32, 4), ("f16", 128, 16, 32, 8), ("f16", 64, 16, 8, 1),
    ("bf16", 128, 16, 64, 8), ("f16", 128, 8, 16, 16),
])
def test_prefill_configurations(oracle, dtype, D, bs, hq, hkv):
    require_gpu()
    b = W.build_prefill_batch("pfcfg", [70, 5, 129, 40], [70, 5, 41, 1], num_heads=hq,
                              num_kv_heads=hkv, head_dim=D, block_size=bs, dtype=dtype,
                              seed=W.BASE_SEED + 741 + D + bs + hq)
    ref, _, _ = _oracle(oracle, b)
    st = PrefillStep(b)
    assert_close(st.run("f32"), ref, dtype, f"prefill {dtype} D{D} bs{bs} G{hq // hkv}")
    assert_no_device_error()


def test_prefill_caches_with_padded_blocks(oracle):
    """Caches whose blocks hold more kv-head slots than the view passed in (a block stride that
    is not num_kv_heads x the head stride) cannot use the one-box-per-tile view of the cache;
    the kernel then reads 8-row boxes.  Same results as the contiguous caches."""
    require_gpu()
    b = W.build_prefill_batch("pfpad", [300, 77, 16, 1, 200], [300, 13, 16, 1, 64], num_heads=32,
                              num_kv_heads=8, head_dim=128, block_size=16, dtype="bf16",
                              seed=W.BASE_SEED + 746)
    ref, kc, vc = _oracle(oracle, b)
    st = PrefillStep(b)
    nb, hkv, bs, d = st.key_cache.shape

    def padded(t):
        big = torch.full((nb, hkv + 1, bs, d), float("nan"), dtype=t.dtype, device=t.device)
        big[:, :hkv] = t
        return big[:, :hkv]

    kpad, vpad = padded(st.key_cache), padded(st.value_cache)
    assert kpad.stride(0) != hkv * kpad.stride(1)
    for dt in ("f32", "bf16"):
        out = torch.full(st.query.shape, float("nan"), dtype=TORCH_DTYPE[dt], device="cuda")
        pa.pa_prefill(out, st.query, kpad, vpad, st.tables, st.lens, st.qs, b.scale, b.block_size,
                      b.num_kv_heads)
        got = to_host(out, dt)
        if dt == "f32":
            assert_close(got, ref, "bf16", "prefill padded-block caches")
        else:
            assert np.array_equal(got, st.run("bf16")), "padded-block caches change the bf16 output"
    assert_no_device_error()


def _scale_keys_by_position(b, factor):
    """Multiply the key of position t of every sequence by factor(t), in the cache and in the
    new tokens' rows, re-rounded to the storage type."""
    dt, bs = b.dtype, b.block_size
    kc = W.decode_to_f64(b.key_cache, dt)
    key = W.decode_to_f64(b.key, dt)
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        q0, q1 = int(b.query_start[s]), int(b.query_start[s + 1])
        for t in range(L - (q1 - q0)):
            kc[b.block_tables[s, t // bs], :, t % bs, :] *= factor(t)
        for j in range(q1 - q0):
            key[q0 + j] *= factor(L - (q1 - q0) + j)
    b.key_cache = W.encode(kc, dt)
    b.key = W.encode(key, dt)


def test_prefill_growing_logits_move_the_reference(oracle):
    """Keys that grow with the position make every later kv tile's logits pass the row's
    reference maximum by far more than 2^8, so the kernel rescales O in tensor memory and takes
    the weights' pass again on almost every tile; the result must not change."""
    require_gpu()
    b = W.build_prefill_batch("pfgrow", [700, 390, 260], [300, 390, 5], num_heads=32,
                              num_kv_heads=8, head_dim=128, block_size=16, dtype="bf16",
                              seed=W.BASE_SEED + 745)
    _scale_keys_by_position(b, lambda t: 1.0 + t / 8.0)
    ref, _, vc = _oracle(oracle, b)
    st = PrefillStep(b)
    assert_close(st.run("f32"), ref, "bf16", "prefill growing logits")
    assert_bf16_output(st.run("bf16"), ref, "prefill growing logits bf16 out", _spread(b, vc, ref))
    assert_no_device_error()


def test_prefill_chunked_workload_full_size(oracle):
    """The full-size chunked-prefill step in the launch configuration the benchmark times;
    the oracle recomputes every sequence (all 2,048 new tokens of all 32 heads)."""
    require_gpu()
    b = W.chunked_prefill()
    st = PrefillStep(b)
    got = st.run("f32")
    gotb = st.run("bf16")
    ref, _, vc = _oracle(oracle, b)
    assert_close(got, ref, "bf16", "chunked prefill (every sequence)")
    assert_bf16_output(gotb, ref, "chunked prefill bf16 out (every sequence)", _spread(b, vc, ref))
    assert_no_device_error()


def test_prefill_single_tokens_match_decode():
    """One new token per sequence is a decode step: pa_prefill and pa_decode agree (two
    kernels, so within the tolerance rather than bit for bit)."""
    require_gpu()
    b = W.build_prefill_batch("pfdec", [17, 300, 1, 64], [1, 1, 1, 1], num_heads=32,
                              num_kv_heads=8, head_dim=128, block_size=16, dtype="bf16",
                              seed=W.BASE_SEED + 742)
    st = PrefillStep(b)
    got = st.run("f32")
    out = torch.empty(st.query.shape, dtype=torch.float32, device="cuda")
    pa.pa_decode(out, st.query, st.key_cache, st.value_cache, st.tables, st.lens, b.scale,
                 b.block_size, b.num_kv_heads)
    assert_close(got, to_host(out, "f32"), "bf16", "prefill vs decode")


def test_prefill_many_small_sequences_use_the_unsorted_schedule(oracle):
    """More (sequence, tile) pairs than the kernel's shared tile list holds (4,096): every CTA
    then takes tiles in sequence order, each warp locating its tile by a scan of query_start.
    4,200 sequences of one to three new tokens on short contexts, one query head per kv head."""
    require_gpu()
    rng = np.random.default_rng(W.BASE_SEED + 747)
    S = 4200
    ql = rng.integers(1, 4, S)
    lens = ql + rng.integers(0, 40, S)
    b = W.build_prefill_batch("pfmany", lens.tolist(), ql.tolist(), num_heads=2, num_kv_heads=2,
                              head_dim=64, block_size=16, dtype="bf16", seed=W.BASE_SEED + 748)
    ref, _, _ = _oracle(oracle, b)
    st = PrefillStep(b)
    assert_close(st.run("f32"), ref, "bf16", "prefill, unsorted schedule")
    assert_no_device_error()


def test_prefill_more_new_tokens_than_context_is_flagged():
    require_gpu()
    b = W.build_prefill_batch("pfbad", [40, 40], [10, 10], num_heads=8, num_kv_heads=2,
                              head_dim=64, block_size=16, dtype="bf16", seed=W.BASE_SEED + 743)
    st = PrefillStep(b)
    st.lens.copy_(torch.tensor([40, 5], dtype=torch.int32))  # sequence 1: 10 new tokens, context 5
    pa.pa_get_device_error(clear=True)
    got = st.run("f32")
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_CONTEXT_LEN
    assert np.all(np.isnan(got[10:20]))      # rows of the bad sequence untouched
    assert np.all(np.isfinite(got[:10]))
