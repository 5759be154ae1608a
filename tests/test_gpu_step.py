"""pa_decode_step: the whole decode step in one call (one kernel when each sequence brings one
new token: the write and the decode fused; otherwise the write, then the decode launched to
overlap it), eagerly, back to back, and captured into a CUDA graph replayed with new inputs."""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import (DeviceBatch, assert_close, assert_no_device_error, oracle_step,
                               require_gpu, to_host, to_torch)

pytestmark = pytest.mark.gpu


def _caches_equal(db, kc, vc, dtype):
    assert np.array_equal(to_host(db.key_cache, dtype).view(np.uint8), kc.view(np.uint8)), "key cache"
    assert np.array_equal(to_host(db.value_cache, dtype).view(np.uint8), vc.view(np.uint8)), "value cache"


def _step(db, out, workspace=None):
    b = db.b
    pa.pa_decode_step(db.key, db.value, db.key_cache, db.value_cache, db.slot_mapping, out,
                      db.query, db.block_tables, db.context_lens, b.scale, b.block_size,
                      b.num_kv_heads, workspace=workspace)


def _workspace(b):
    ws = torch.empty(pa.pa_decode_workspace_bytes(b.num_seqs, b.num_heads, b.num_kv_heads,
                                                  b.head_dim, 0), dtype=torch.uint8, device="cuda")
    pa.pa_workspace_init(ws)
    return ws


@pytest.mark.parametrize("own_workspace", [False, True])
def test_step_equals_write_then_decode(oracle, own_workspace):
    require_gpu()
    b = W.llama3_8b_decode(num_seqs=24, min_len=1, max_len=2048)
    ref, kc, vc = oracle_step(oracle, b)
    db = DeviceBatch(b)
    out = torch.full(db.query.shape, float("nan"), dtype=torch.float32, device="cuda")
    _step(db, out, _workspace(b) if own_workspace else None)
    _caches_equal(db, kc, vc, "bf16")
    assert_close(to_host(out, "f32"), ref, "bf16", "pa_decode_step")
    assert_no_device_error()


def test_step_refuses_before_launching():
    require_gpu()
    b = W.llama3_8b_decode(num_seqs=4, min_len=1, max_len=100)
    db = DeviceBatch(b)
    before = db.key_cache.clone()
    out = torch.zeros(db.query.shape, dtype=torch.float32, device="cuda")
    bad_lens = db.context_lens[:3].clone()  # one length short: the decode half is refused
    with pytest.raises(pa.PagedAttentionError) as info:
        pa.pa_decode_step(db.key, db.value, db.key_cache, db.value_cache, db.slot_mapping, out,
                          db.query, db.block_tables, bad_lens, b.scale, b.block_size,
                          b.num_kv_heads)
    assert info.value.status == pa.PA_ERR_SHAPE
    torch.cuda.synchronize()
    # the write half did not run either (bytes compared: unused slots hold NaN)
    assert torch.equal(db.key_cache.view(torch.int16), before.view(torch.int16))
    assert torch.all(out == 0)


def test_step_in_cuda_graph_replays_with_new_inputs(oracle):
    """Capture one step with a caller workspace, then replay it for three batches of the same
    shapes copied into the captured tensors; each replay matches the oracle for its batch."""
    require_gpu()
    make = [lambda k=k: W.build_batch(
        "graph", W.llama3_8b_decode(num_seqs=16, min_len=1, max_len=1500).context_lens,
        num_heads=32, num_kv_heads=8, head_dim=128, block_size=16, dtype="bf16",
        seed=W.BASE_SEED + 700 + k, max_blocks=128) for k in range(3)]
    batches = [m() for m in make]
    db = DeviceBatch(batches[0])
    ws = _workspace(batches[0])
    out = torch.empty(db.query.shape, dtype=torch.float32, device="cuda")
    _step(db, out, ws)  # eager first: kernels and descriptors prepared outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _step(db, out, ws)
    for b in batches:
        ref, kc, vc = oracle_step(oracle, b)
        src = DeviceBatch(b)
        for name in ("query", "key", "value", "slot_mapping", "block_tables", "context_lens",
                     "key_cache", "value_cache"):
            getattr(db, name).copy_(getattr(src, name))
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        _caches_equal(db, kc, vc, "bf16")
        assert_close(to_host(out, "f32"), ref, "bf16", "graph replay")
    del g
    assert_no_device_error()


def test_consecutive_fused_steps_read_the_previous_steps_write(oracle):
    """Two steps on one pool, launched back to back: step 1 brings token L-1 of each sequence
    (written by its kernel), step 2 token L with one more position of context, so step 2 reads
    position L-1 from the cache that step 1's kernel wrote.  Both outputs against the oracle."""
    require_gpu()
    lens = W.llama3_8b_decode(num_seqs=20, min_len=2, max_len=1200).context_lens.astype(np.int32)
    b = W.build_batch("two_steps", lens + 1, num_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=16, dtype="bf16", seed=W.BASE_SEED + 780, keep_logical=True)
    S, bs = b.num_seqs, b.block_size
    slot = lambda s, t: int(b.block_tables[s, t // bs]) * bs + t % bs  # noqa: E731
    kc0, vc0 = b.key_cache.copy(), b.value_cache.copy()
    for s in range(S):  # position L-1 arrives with step 1: not in the pool yet
        p = slot(s, int(lens[s]) - 1)
        kc0[p // bs, :, p % bs, :] = 0xFFFF
        vc0[p // bs, :, p % bs, :] = 0xFFFF
    steps = []
    for k, t_new in ((1, lens - 1), (2, lens)):
        key = np.stack([b.logical_key[s][t_new[s]] for s in range(S)])
        value = np.stack([b.logical_value[s][t_new[s]] for s in range(S)])
        slots = np.array([slot(s, int(t_new[s])) for s in range(S)], np.int64)
        steps.append((key, value, slots, (t_new + 1).astype(np.int32)))
    dev = lambda x, dt=None: to_torch(x, dt)  # noqa: E731
    kc, vc = dev(kc0, "bf16"), dev(vc0, "bf16")
    q, tables = dev(b.query, "bf16"), dev(b.block_tables)
    ws = _workspace(b)
    outs = []
    for key, value, slots, ctx in steps:  # no synchronisation between the two steps
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        pa.pa_decode_step(dev(key, "bf16"), dev(value, "bf16"), kc, vc, dev(slots), out, q,
                          tables, dev(ctx), b.scale, bs, b.num_kv_heads, workspace=ws)
        outs.append(out)
    torch.cuda.synchronize()
    hk, hv = kc0.copy(), vc0.copy()
    for (key, value, slots, ctx), out in zip(steps, outs):
        assert oracle.reshape_and_cache(key, value, hk, hv, slots, "bf16") == 0
        ref = oracle.decode(b.query, hk, hv, b.block_tables, ctx, b.scale, "bf16")
        assert_close(to_host(out, "f32"), ref, "bf16", "consecutive fused steps")
    assert np.array_equal(to_host(kc, "bf16").view(np.uint8), hk.view(np.uint8))
    assert np.array_equal(to_host(vc, "bf16").view(np.uint8), hv.view(np.uint8))
    assert_no_device_error()


def test_fused_step_flags_a_slot_that_is_not_the_last_position(oracle):
    """Token s must be sequence s's position L-1: a slot elsewhere is stored as asked but
    flagged (PA_DEVERR_SLOT); the other sequences are unaffected."""
    require_gpu()
    b = W.llama3_8b_decode(num_seqs=6, min_len=40, max_len=300)
    used = set()
    for s in range(b.num_seqs):
        used.update(int(x) for x in b.block_tables[s, :(int(b.context_lens[s]) + 15) // 16])
    free = next(i for i in range(b.num_blocks) if i not in used)
    b.slot_mapping[3] = free * b.block_size  # a free block, not sequence 3's position L-1
    db = DeviceBatch(b)
    out = torch.full(db.query.shape, float("nan"), dtype=torch.float32, device="cuda")
    pa.pa_get_device_error(clear=True)
    _step(db, out)
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_SLOT
    ref, kc, vc = oracle_step(oracle, b)
    _caches_equal(db, kc, vc, "bf16")
    keep = [s for s in range(b.num_seqs) if s != 3]
    assert_close(to_host(out, "f32")[keep], ref[keep], "bf16", "other sequences")


def test_step_with_more_new_tokens_than_sequences(oracle):
    """The shared-prefix batch writes several tokens per sequence: the write kernel, then the
    decode (two kernels), against the oracle."""
    require_gpu()
    b = W.shared_prefix(num_groups=4, suffix_range=(16, 200))
    assert len(b.slot_mapping) > b.num_seqs
    ref, kc, vc = oracle_step(oracle, b)
    db = DeviceBatch(b)
    pa.pa_copy_blocks(db.key_cache, db.value_cache, db.block_mapping)
    out = torch.full(db.query.shape, float("nan"), dtype=torch.float32, device="cuda")
    _step(db, out)
    _caches_equal(db, kc, vc, "bf16")
    assert_close(to_host(out, "f32"), ref, "bf16", "two-kernel step")
    assert_no_device_error()
