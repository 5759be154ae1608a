"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (code running under CUDA graph capture, engines that reserve all device memory up
front, latency-critical loops that cannot take an allocation's implicit synchronisation) use
pa_decode_noalloc, whose scratch is a fixed array inside the library.  These tests call it
through the C ABI twice in a row and compare each result with the existing pa_decode entry
point, within the parity tolerance for bf16 caches with fp32 output; the second call checks that
the scratch left by the first does not disturb the next one.  This file is collected last so a
run that stops at the first failure has run every other test already; it also passes when run
alone in a fresh process (the first call on the device sets the scratch up).
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import DeviceBatch, assert_close, assert_no_device_error, require_gpu, to_host

pytestmark = pytest.mark.gpu


def _noalloc(db, out):
    b = db.b
    pa.pa_decode_noalloc(out, db.query, db.key_cache, db.value_cache, db.block_tables,
                         db.context_lens, b.scale, b.block_size, b.num_kv_heads)


@pytest.mark.parametrize("batch", [
    lambda: W.llama3_8b_decode(num_seqs=24, min_len=1, max_len=2048),
    # one long context split over many warps (merges) next to short ones
    lambda: W.build_batch("mixed", [20000, 3, 700, 1, 0, 129], num_heads=32, num_kv_heads=8,
                          head_dim=128, block_size=16, dtype="bf16", seed=W.BASE_SEED + 990),
])
def test_noalloc_matches_pa_decode_on_two_calls(batch):
    require_gpu()
    b = batch()
    db = DeviceBatch(b)
    db.write()
    ref = to_host(db.decode("f32"), "f32")  # the existing entry point, pa_decode
    for call in range(2):
        out = torch.full(db.query.shape, float("nan"), dtype=torch.float32, device="cuda")
        _noalloc(db, out)
        assert_close(to_host(out, "f32"), ref, "bf16", f"pa_decode_noalloc call {call + 1}")
    assert_no_device_error()


def test_noalloc_refuses_shapes_beyond_its_scratch():
    require_gpu()
    S = 4096  # 32768 (sequence, kv head) pairs: far more scratch than the fixed array holds
    b = W.build_batch("wide", np.ones(S, np.int32), num_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=16, dtype="bf16", seed=W.BASE_SEED + 991)
    db = DeviceBatch(b)
    out = torch.zeros(db.query.shape, dtype=torch.float32, device="cuda")
    with pytest.raises(pa.PagedAttentionError) as info:
        _noalloc(db, out)
    assert info.value.status == pa.PA_ERR_WORKSPACE
    assert "static scratch" in str(info.value)
    assert torch.all(out == 0)  # nothing was launched
