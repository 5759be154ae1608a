"""pa_decode_shared_prefix against the oracle: groups of sequences whose block tables name the same
physical blocks for a common prompt prefix ([P2] 4.1, [P3] 2.2).  The result is the plain
decode of each sequence (the oracle's definition); the cascade only changes the order of the
arithmetic, so the tolerances are those of pa_decode (tests/gpu_helpers.py).
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import (TORCH_DTYPE, DeviceBatch, assert_bf16_output, assert_close,
                               assert_no_device_error, oracle_step, require_gpu, to_host,
                               to_torch, value_spread)

pytestmark = pytest.mark.gpu


def _shared(db, groups, prefixes, out_dtype="f32", workspace=None):
    b = db.b
    out = torch.full(db.query.shape, float("nan"), dtype=TORCH_DTYPE[out_dtype], device="cuda")
    pa.pa_decode_shared_prefix(out, db.query, db.key_cache, db.value_cache, db.block_tables,
                               db.context_lens, to_torch(groups), to_torch(prefixes), b.scale,
                               b.block_size, b.num_kv_heads, workspace=workspace)
    return to_host(out, out_dtype)


def _share_prefixes(b, sizes, prefix):
    """Make the consecutive groups of `sizes` members share their first member's blocks for
    the first prefix[g] positions (the members' own blocks there go unused).  Returns
    (group_start, prefix_lens)."""
    starts = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    lens = np.zeros(b.num_seqs, np.int32)
    for g in range(len(sizes)):
        first, end = int(starts[g]), int(starts[g + 1])
        nb = prefix[g] // b.block_size
        for s in range(first, end):
            b.block_tables[s, :nb] = b.block_tables[first, :nb]
            lens[s] = prefix[g]
    return starts, lens


def test_shared_prefix_workload_every_sequence(oracle):
    """The full-size shared-prefix batch (128 sequences sharing a 1024-token prompt) after its
    copy-on-write and writes, fp32 and bf16 out, every sequence against the oracle."""
    require_gpu()
    b = W.shared_prefix()
    groups, prefixes = W.shared_groups(b)
    db = DeviceBatch(b)
    db.write()
    ref, kc, vc = oracle_step(oracle, b)
    got = _shared(db, groups, prefixes)
    assert_close(got, ref, "bf16", "shared prefix cascade (every sequence)")
    gotb = _shared(db, groups, prefixes, "bf16")
    assert_bf16_output(gotb, ref, "shared prefix cascade bf16",
                       value_spread(vc, b.dtype, b.block_tables, b.context_lens, ref, b.block_size))
    assert_no_device_error()


@pytest.mark.parametrize("dtype,D,bs,hq,hkv", [
    ("bf16", 128, 16, 32, 8), ("bf16", 128, 8, 8, 8), ("bf16", 64, 32, 16, 8),
    ("f16", 128, 32, 16, 2), ("bf16", 64, 16, 8, 1), ("f16", 64, 8, 32, 4),
])
def test_groups_of_several_sizes_and_prefixes(oracle, dtype, D, bs, hq, hkv):
    """Groups of 1, 3, 40 and 7 members with prefixes of 0, one block, 512 and 1088 positions
    (one to five prefix items), a member whose context ends inside the prefix (decoded whole),
    and every member's suffix of its own."""
    require_gpu()
    rng = np.random.default_rng([D, bs, hq])
    sizes = [1, 3, 40, 7]
    prefix = [0, bs, 512, 1088]
    lens = []
    for g, n in enumerate(sizes):
        lens += list(prefix[g] + rng.integers(1, 300, n))
    lens = np.array(lens, np.int32)
    lens[5] = 300  # group 2's first member ends inside its group's 512-position prefix
    b = W.build_batch("shared", lens, num_heads=hq, num_kv_heads=hkv, head_dim=D, block_size=bs,
                      dtype=dtype, seed=W.BASE_SEED + 960 + D + bs)
    groups, prefixes = _share_prefixes(b, sizes, prefix)
    db = DeviceBatch(b)
    db.write()
    ref, _, _ = oracle_step(oracle, b)
    what = f"shared {dtype} D{D} bs{bs} G{hq // hkv}"
    assert_close(_shared(db, groups, prefixes), ref, dtype, what)
    # the same step again with a caller workspace: the merge counters are left ready
    n = pa.pa_decode_shared_prefix_workspace_bytes(b.num_seqs, hq, hkv, D, b.max_blocks, bs)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        assert_close(_shared(db, groups, prefixes, workspace=ws), ref, dtype, what + " (caller workspace)")
    assert_no_device_error()


def test_disagreeing_members_are_flagged(oracle):
    """A prefix that is not a whole number of blocks is decoded whole (correct, flagged); a
    member naming other blocks or another prefix length than its first member is flagged."""
    require_gpu()
    lens = np.array([700, 650, 800, 720], np.int32)
    b = W.build_batch("shared_bad", lens, num_heads=32, num_kv_heads=8, head_dim=128,
                      block_size=16, dtype="bf16", seed=W.BASE_SEED + 970)
    groups, prefixes = _share_prefixes(b, [4], [512])
    db = DeviceBatch(b)
    db.write()
    ref, _, _ = oracle_step(oracle, b)
    pa.pa_get_device_error(clear=True)
    odd = prefixes.copy()
    odd[:] = 504  # not a multiple of the block size: every member decodes its whole context
    assert_close(_shared(db, groups, odd), ref, "bf16", "prefix of a partial block, decoded whole")
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_PREFIX
    mismatch = prefixes.copy()
    mismatch[2] = 256
    _shared(db, groups, mismatch)
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_PREFIX
    assert_close(_shared(db, groups, prefixes), ref, "bf16", "agreeing members again")
    assert_no_device_error()


def test_no_sharing_is_the_plain_decode(oracle):
    """One group per sequence, nothing shared: the decode kernel alone, as pa_decode."""
    require_gpu()
    b = W.llama3_8b_decode(num_seqs=10, min_len=1, max_len=400)
    groups, prefixes = W.shared_groups(b)
    db = DeviceBatch(b)
    db.write()
    ref, _, _ = oracle_step(oracle, b)
    assert_close(_shared(db, groups, prefixes), ref, "bf16", "no shared prefix")
    assert_no_device_error()
