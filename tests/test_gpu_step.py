"""pa_decode_step: the whole decode step (cache write, then decode launched to overlap it) in
one call, eagerly and captured into a CUDA graph that is replayed with new inputs."""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import (DeviceBatch, assert_close, assert_no_device_error, oracle_step,
                               require_gpu, to_host)

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
