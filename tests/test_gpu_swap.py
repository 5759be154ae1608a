"""pa_swap_blocks: block-level swap between the device cache and a cache in pinned host memory
(swap out, reuse of the device blocks, swap back in elsewhere), checked byte for byte against
the oracle and through the decode that follows."""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import DeviceBatch, assert_no_device_error, require_gpu, to_host

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def test_swap_out_reuse_swap_in(oracle):
    require_gpu()
    b = W.llama3_8b_decode(num_seqs=12, min_len=100, max_len=1200)
    db = DeviceBatch(b)
    db.write()
    before = to_host(db.decode("f32"), "f32")
    kc_host_view = to_host(db.key_cache, "bf16").copy()
    vc_host_view = to_host(db.value_cache, "bf16").copy()

    nb = b.num_blocks
    nh = 600
    rng = np.random.default_rng(5)
    hk = torch.empty((nh,) + tuple(db.key_cache.shape[1:]), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    hk.view(torch.int16).copy_(torch.from_numpy(rng.integers(-2**15, 2**15, hk.shape, dtype=np.int16)))
    hv.view(torch.int16).copy_(torch.from_numpy(rng.integers(-2**15, 2**15, hv.shape, dtype=np.int16)))
    hk0 = hk.view(torch.int16).numpy().view(np.uint16).copy()
    hv0 = hv.view(torch.int16).numpy().view(np.uint16).copy()

    # swap out sequences 3 and 7: every block of their tables, to scattered host blocks
    seqs = [3, 7]
    dev_ids = np.concatenate([b.block_tables[s, :-(-int(b.context_lens[s]) // b.block_size)]
                              for s in seqs]).astype(np.int64)
    host_ids = rng.permutation(nh)[:len(dev_ids)].astype(np.int64)
    pairs = torch.from_numpy(np.stack([dev_ids, host_ids], 1)).cuda()
    pa.pa_swap_blocks(db.key_cache, db.value_cache, hk, hv, pairs)
    torch.cuda.synchronize()
    ek, ev = hk0.copy(), hv0.copy()
    assert oracle.swap_blocks(kc_host_view.view(np.uint16), vc_host_view.view(np.uint16), ek, ev,
                              pairs.cpu().numpy(), "bf16") == 0
    assert np.array_equal(hk.view(torch.int16).numpy().view(np.uint16), ek)
    assert np.array_equal(hv.view(torch.int16).numpy().view(np.uint16), ev)

    # the device blocks go to someone else: overwrite them
    idx = torch.from_numpy(dev_ids).cuda()
    db.key_cache[idx] = float("nan")
    db.value_cache[idx] = float("nan")
    # swap back in to other free device blocks (the mapping itself in pinned host memory)
    used = set()
    for s in range(b.num_seqs):
        used |= set(b.block_tables[s, :-(-int(b.context_lens[s]) // b.block_size)].tolist())
    free = np.array(sorted(set(range(nb)) - used), np.int64)
    new_ids = rng.permutation(free)[:len(dev_ids)]
    back = torch.from_numpy(np.stack([host_ids, new_ids], 1)).pin_memory()
    pa.pa_swap_blocks(hk, hv, db.key_cache, db.value_cache, back)
    tables = b.block_tables.copy()
    at = 0
    for s in seqs:
        n = -(-int(b.context_lens[s]) // b.block_size)
        tables[s, :n] = new_ids[at:at + n]
        at += n
    db.block_tables.copy_(torch.from_numpy(tables))
    after = to_host(db.decode("f32"), "f32")
    assert np.array_equal(after, before)  # same logical K/V, other physical blocks: same bits
    assert_no_device_error()


def test_swap_between_device_pools_and_bad_ids():
    require_gpu()
    src_k = torch.randn(40, 8, 16, 128, device="cuda").to(torch.bfloat16)
    src_v = torch.randn_like(src_k)
    dst_k = torch.zeros(10, 8, 16, 128, dtype=torch.bfloat16, device="cuda")
    dst_v = torch.zeros_like(dst_k)
    pairs = torch.tensor([[39, 0], [5, 9], [0, 4]], dtype=torch.int64, device="cuda")
    pa.pa_swap_blocks(src_k, src_v, dst_k, dst_v, pairs)
    for s, d in pairs.tolist():
        assert torch.equal(_bits(dst_k[d]), _bits(src_k[s])) and torch.equal(_bits(dst_v[d]), _bits(src_v[s]))
    untouched = [i for i in range(10) if i not in (0, 9, 4)]
    assert torch.all(dst_k[untouched] == 0)
    assert pa.pa_get_device_error(clear=True) == 0
    bad = torch.tensor([[40, 1], [2, 10], [-1, 2]], dtype=torch.int64, device="cuda")
    snap = dst_k.clone()
    pa.pa_swap_blocks(src_k, src_v, dst_k, dst_v, bad)
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_COPY_PAIR
    assert torch.equal(_bits(dst_k), _bits(snap))


def test_swap_refuses_pageable_host_memory():
    require_gpu()
    dk = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16, device="cuda")
    hk = torch.zeros(4, 2, 16, 64, dtype=torch.bfloat16)  # pageable
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    with pytest.raises(pa.PagedAttentionError) as info:
        pa.pa_swap_blocks(dk, dk, hk, hk, pairs)
    assert info.value.status == pa.PA_ERR_LAYOUT
    other = torch.zeros(4, 2, 8, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pa.PagedAttentionError) as info:
        pa.pa_swap_blocks(dk, dk, other, other, pairs)
    assert info.value.status == pa.PA_ERR_SHAPE
