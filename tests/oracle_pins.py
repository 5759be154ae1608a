"""Pins for the CPU oracle: checks against facts that do not come from the oracle itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when the oracle disagrees with:
  * brute force: contiguous attention straight from the generator's logical K/V streams (no
    block table, no max subtraction, numpy long double);
  * a library routine: torch's scaled_dot_product_attention in float64 on the CPU;
  * closed forms: one token, constant values, zero query, a dominant key, two tokens, and a
    three-token example evaluated with Python's decimal module;
  * invariants the sources fix: placement of physical blocks, block size, unread slots and
    block-table entries, shared blocks, and the split-context merge.
The same pins run against deliberately broken copies of the oracle (test_oracle_mutants.py);
each broken copy must fail at least one of them.

Sources (vLLM tutorials): [P2] "vLLM core features: PagedAttention, Continuous Batching,
quantization support, distributed inference" 4.1; [P3] "Core inference engine (part 1): vLLM
architecture, PagedAttention principle, Continuous Batching mechanism" 2.2; [P4] "vLLM core
architecture: model loading, PagedAttention principle, KV cache management" 2.2.1, 2.2.2.
"""
from __future__ import annotations

import math
from decimal import Decimal, getcontext

import numpy as np

from paged_kv_cache_427_b200 import workloads as W

REL_TOL_F64 = 1e-12


def _rel_err(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = max(1e-300, float(np.max(np.abs(b))) if b.size else 1.0)
    return float(np.max(np.abs(a - b))) / scale if a.size else 0.0


def _step(orc, batch: W.PagedBatch):
    """Run the oracle's step on copies of the pool: copies, writes, then decode."""
    kc = batch.key_cache.copy()
    vc = batch.value_cache.copy()
    if batch.block_mapping is not None and len(batch.block_mapping):
        assert orc.copy_blocks(kc, vc, batch.block_mapping, batch.dtype) == 0
    assert orc.reshape_and_cache(batch.key, batch.value, kc, vc, batch.slot_mapping,
                                 batch.dtype) == 0
    out = orc.decode(batch.query, kc, vc, batch.block_tables, batch.context_lens, batch.scale,
                     batch.dtype)
    return out, kc, vc


def brute_force(batch: W.PagedBatch) -> np.ndarray:
    """Attention over the logical streams, long double, no max subtraction, no paging."""
    S, Hq, D = batch.query.shape
    G = Hq // batch.num_kv_heads
    out = np.zeros((S, Hq, D), dtype=np.longdouble)
    for s in range(S):
        L = int(batch.context_lens[s])
        if L <= 0:
            continue
        K = W.decode_to_f64(batch.logical_key[s][:L], batch.dtype).astype(np.longdouble)
        V = W.decode_to_f64(batch.logical_value[s][:L], batch.dtype).astype(np.longdouble)
        q = W.decode_to_f64(batch.query[s], batch.dtype).astype(np.longdouble)
        for h in range(Hq):
            g = h // G
            z = np.longdouble(batch.scale) * np.einsum("td,d->t", K[:, g, :], q[h])
            w = np.exp(z)
            out[s, h] = np.einsum("t,td->d", w, V[:, g, :]) / w.sum()
    return out


def _small_batches():
    """Tiny structured cases: several G, D, block sizes and element types."""
    cases = []
    rng = np.random.default_rng([W.BASE_SEED, 99])
    specs = [  # (Hq, Hkv, D, bs, dtype)
        (4, 4, 64, 16, "f32"),
        (8, 2, 64, 8, "bf16"),
        (8, 2, 128, 32, "bf16"),
        (4, 1, 128, 16, "f32"),
        (6, 3, 64, 8, "f16"),
    ]
    for i, (hq, hkv, d, bs, dt) in enumerate(specs):
        lens = rng.integers(1, 100, size=5).astype(np.int32)
        lens[0] = 1
        lens[1] = bs          # exactly one full block
        lens[2] = bs + 1      # one token into the second block
        cases.append(W.build_batch(f"small{i}", lens, num_heads=hq, num_kv_heads=hkv,
                                   head_dim=d, block_size=bs, dtype=dt,
                                   seed=W.BASE_SEED + 100 + i, keep_logical=True))
    cases.append(W.tiny_fp32())
    return cases


# ---------------------------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------------------------

def pin_brute_force(orc):
    """The paged oracle equals contiguous long-double attention on the logical streams."""
    for batch in _small_batches():
        out, _, _ = _step(orc, batch)
        ref = brute_force(batch)
        err = _rel_err(out, ref.astype(np.float64))
        assert err < REL_TOL_F64, f"{batch.name}: brute-force rel err {err:.3e}"


def pin_torch_sdpa(orc):
    """The oracle equals torch.nn.functional.scaled_dot_product_attention (float64, CPU)."""
    import torch

    for batch in _small_batches():
        out, _, _ = _step(orc, batch)
        S, Hq, D = batch.query.shape
        for s in range(S):
            L = int(batch.context_lens[s])
            K = torch.from_numpy(W.decode_to_f64(batch.logical_key[s][:L], batch.dtype))
            V = torch.from_numpy(W.decode_to_f64(batch.logical_value[s][:L], batch.dtype))
            q = torch.from_numpy(W.decode_to_f64(batch.query[s], batch.dtype))
            ref = torch.nn.functional.scaled_dot_product_attention(
                q[:, None, :], K.permute(1, 0, 2), V.permute(1, 0, 2), scale=batch.scale,
                enable_gqa=True)[:, 0, :].numpy()
            err = _rel_err(out[s], ref)
            assert err < REL_TOL_F64, f"{batch.name} seq {s}: sdpa rel err {err:.3e}"


def _custom(context_lens, key_rows, value_rows, query, *, Hq, Hkv, D, bs=16, dtype="f32",
            scale=None):
    """A batch from explicit logical rows ([S] lists of [L, Hkv, D] float arrays)."""
    b = W.build_batch("custom", context_lens, num_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                      block_size=bs, dtype=dtype, seed=W.BASE_SEED + 500, keep_logical=True)
    kc = W._fill_pool(b.key_cache.shape, dtype, "nan")
    vc = W._fill_pool(b.value_cache.shape, dtype, "nan")
    for s, L in enumerate(context_lens):
        kr = W.encode(np.asarray(key_rows[s], np.float32), dtype)
        vr = W.encode(np.asarray(value_rows[s], np.float32), dtype)
        W._place(kc, b.block_tables[s], 0, kr[:L - 1], bs)
        W._place(vc, b.block_tables[s], 0, vr[:L - 1], bs)
        b.key[s], b.value[s] = kr[L - 1], vr[L - 1]
        b.logical_key[s], b.logical_value[s] = kr, vr
    b.key_cache, b.value_cache = kc, vc
    b.query = W.encode(np.asarray(query, np.float32), dtype)
    if scale is not None:
        b.scale = scale
    return b


def pin_closed_forms(orc):
    """One token -> its value row; equal values -> that value; zero query or equal keys -> mean;
    a dominant key -> its value row; two tokens -> the logistic mix."""
    rng = np.random.default_rng(7)
    Hq, Hkv, D = 4, 2, 64
    # (a) context of one token: the output is that token's value row, exactly.
    k1 = [rng.standard_normal((1, Hkv, D)).astype(np.float32) for _ in range(3)]
    v1 = [rng.standard_normal((1, Hkv, D)).astype(np.float32) for _ in range(3)]
    q = rng.standard_normal((3, Hq, D)).astype(np.float32)
    b = _custom([1, 1, 1], k1, v1, q, Hq=Hq, Hkv=Hkv, D=D)
    out, _, _ = _step(orc, b)
    for s in range(3):
        for h in range(Hq):
            assert np.array_equal(out[s, h], v1[s][0, h // 2].astype(np.float64)), "L=1"
    # (b) all value rows equal c -> output c.
    L = 41
    kk = [rng.standard_normal((L, Hkv, D)).astype(np.float32)]
    c = rng.standard_normal((Hkv, D)).astype(np.float32)
    vv = [np.broadcast_to(c, (L, Hkv, D)).copy()]
    b = _custom([L], kk, vv, rng.standard_normal((1, Hq, D)), Hq=Hq, Hkv=Hkv, D=D)
    out, _, _ = _step(orc, b)
    for h in range(Hq):
        assert _rel_err(out[0, h], c[h // 2]) < 1e-15, "constant V"
    # (c) zero query -> mean of V; (d) equal keys -> mean of V.
    vv = [rng.standard_normal((L, Hkv, D)).astype(np.float32)]
    mean = vv[0].astype(np.float64).mean(axis=0)
    b = _custom([L], kk, vv, np.zeros((1, Hq, D)), Hq=Hq, Hkv=Hkv, D=D)
    out, _, _ = _step(orc, b)
    for h in range(Hq):
        assert _rel_err(out[0, h], mean[h // 2]) < 1e-13, "zero query"
    keq = [np.broadcast_to(rng.standard_normal((1, Hkv, D)).astype(np.float32),
                           (L, Hkv, D)).copy()]
    b = _custom([L], keq, vv, rng.standard_normal((1, Hq, D)), Hq=Hq, Hkv=Hkv, D=D)
    out, _, _ = _step(orc, b)
    for h in range(Hq):
        assert _rel_err(out[0, h], mean[h // 2]) < 1e-13, "equal keys"
    # (e) one key whose logit leads every other by more than 60 -> its value row.
    qd = np.zeros((1, Hq, D), np.float32)
    qd[0, :, 0] = 1.0
    kd = np.zeros((L, Hkv, D), np.float32)
    kd[:, :, 1:] = rng.standard_normal((L, Hkv, D - 1))
    j = 29
    kd[j, :, 0] = 512.0  # scale 1/8 -> logit 64, others 0
    b = _custom([L], [kd], vv, qd, Hq=Hq, Hkv=Hkv, D=D, scale=1.0 / 8)
    out, _, _ = _step(orc, b)
    for h in range(Hq):
        assert _rel_err(out[0, h], vv[0][j, h // 2]) < 1e-20 * L + 1e-26, "dominant key"
    # (f) two tokens: out = s(z0 - z1) v0 + s(z1 - z0) v1 with s the logistic function.
    q2 = np.zeros((1, Hq, D), np.float32)
    q2[0, :, 0] = 2.0
    k2 = np.zeros((2, Hkv, D), np.float32)
    k2[0, :, 0] = 0.75
    k2[1, :, 0] = -1.25
    v2 = rng.standard_normal((2, Hkv, D)).astype(np.float32)
    b = _custom([2], [k2], [v2], q2, Hq=Hq, Hkv=Hkv, D=D, scale=0.5)
    out, _, _ = _step(orc, b)
    z0, z1 = 0.5 * 2.0 * 0.75, 0.5 * 2.0 * -1.25
    s01 = 1.0 / (1.0 + math.exp(z1 - z0))
    for h in range(Hq):
        ref = s01 * v2[0, h // 2].astype(np.float64) + (1 - s01) * v2[1, h // 2].astype(np.float64)
        assert _rel_err(out[0, h], ref) < 1e-15, "two tokens"


def pin_decimal_example(orc):
    """Three tokens with logits {0, 1, -2} (exact in binary), values evaluated with 40-digit
    decimal arithmetic; the context straddles a block boundary (block_size 2)."""
    getcontext().prec = 40
    Hq = Hkv = 1
    D = 64
    q = np.zeros((1, 1, D), np.float32)
    q[0, 0, 0] = 1.0
    k = np.zeros((3, 1, D), np.float32)
    k[:, 0, 0] = [0.0, 1.0, -2.0]
    v = np.zeros((3, 1, D), np.float32)
    v[:, 0, 0] = [1.0, 2.0, 4.0]
    v[:, 0, 1] = [-3.0, 0.5, 8.0]
    b = _custom([3], [k], [v], q, Hq=Hq, Hkv=Hkv, D=D, bs=8, scale=1.0)
    b2 = W.build_batch("custom", [3], num_heads=1, num_kv_heads=1, head_dim=D, block_size=2,
                       dtype="f32", seed=1, keep_logical=True)
    kc = W._fill_pool(b2.key_cache.shape, "f32", "nan")
    vc = W._fill_pool(b2.value_cache.shape, "f32", "nan")
    W._place(kc, b2.block_tables[0], 0, k, 2)
    W._place(vc, b2.block_tables[0], 0, v, 2)
    for batch, caches in ((b, None), (b2, (kc, vc))):
        if caches is None:
            out, _, _ = _step(orc, batch)
        else:
            out = orc.decode(q, caches[0], caches[1], b2.block_tables, np.array([3], np.int32),
                             1.0, "f32")
        e = [Decimal(z).exp() for z in (0, 1, -2)]
        den = sum(e)
        exp0 = (e[0] * 1 + e[1] * 2 + e[2] * 4) / den
        exp1 = (e[0] * Decimal(-3) + e[1] * Decimal("0.5") + e[2] * 8) / den
        assert abs(Decimal(float(out[0, 0, 0])) - exp0) < Decimal("1e-15"), "decimal d0"
        assert abs(Decimal(float(out[0, 0, 1])) - exp1) < Decimal("1e-15"), "decimal d1"
        assert np.all(out[0, 0, 2:] == 0.0), "decimal zeros"


def pin_placement_invariance(orc):
    """[P4] 2.2.1: physical blocks may sit anywhere.  Same logical values, other permutation or
    other block size (8/16/32), unread slots poisoned or zeroed -> bit-identical output."""
    lens = np.array([1, 7, 8, 9, 33, 70], np.int32)
    outs = []
    for bs in (8, 16, 32):
        for salt in (0, 1):
            for fill in ("nan", "zero"):
                b = W.build_batch("inv", lens, num_heads=8, num_kv_heads=2, head_dim=64,
                                  block_size=bs, dtype="bf16", seed=W.BASE_SEED + 700,
                                  perm_salt=salt, fill=fill, pool_factor=2.0)
                outs.append(_step(orc, b)[0])
    for o in outs[1:]:
        assert np.array_equal(o, outs[0]), "placement / block size changed the output"


def pin_unread_table_entries(orc):
    """Block-table entries past a sequence's last block are never read, however invalid."""
    b = W.build_batch("tab", [5, 17, 40], num_heads=4, num_kv_heads=2, head_dim=64,
                      block_size=16, dtype="bf16", seed=W.BASE_SEED + 701, max_blocks=6)
    ref, _, _ = _step(orc, b)
    t = b.block_tables.copy()
    t[t < 0] = 2 ** 30
    b.block_tables = t
    out, _, _ = _step(orc, b)
    assert np.array_equal(out, ref), "entries past the context changed the output"


def pin_cache_write(orc):
    """[P2] 4.1: a new token lands at offset slot % bs of block slot / bs.  Reading every
    sequence back through its block table gives its logical stream; nothing else changes;
    negative slots store nothing; slots outside the pool are refused."""
    for batch in _small_batches() + [W.shared_prefix(num_groups=3, suffix_range=(16, 60),
                                                     keep_logical=True)]:
        _, kc, vc = _step(orc, batch)
        bs = batch.block_size
        for s in range(batch.num_seqs):
            L = int(batch.context_lens[s])
            t = np.arange(L)
            phys = batch.block_tables[s][t // bs]
            got_k = kc[phys, :, t % bs, :]
            got_v = vc[phys, :, t % bs, :]
            assert np.array_equal(got_k.view(np.uint8), batch.logical_key[s][:L].view(np.uint8))
            assert np.array_equal(got_v.view(np.uint8), batch.logical_value[s][:L].view(np.uint8))
        # bytes outside the written slots and the copied blocks are untouched
        touched = np.zeros(kc.shape[:1] + kc.shape[2:3], bool)
        for sl in batch.slot_mapping:
            touched[sl // bs, sl % bs] = True
        if batch.block_mapping is not None:
            for _, dst in batch.block_mapping:
                touched[dst, :] = True
        keep = ~touched
        a = kc.transpose(0, 2, 1, 3)[keep]
        b0 = batch.key_cache.transpose(0, 2, 1, 3)[keep]
        assert np.array_equal(a.view(np.uint8), b0.view(np.uint8)), "untouched slots changed"
    b = W.tiny_fp32()
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    slots = b.slot_mapping.copy()
    slots[1] = -1                               # padding token: stores nothing
    slots[2] = b.num_blocks * b.block_size      # first slot past the pool: refused
    skipped = orc.reshape_and_cache(b.key, b.value, kc, vc, slots, "f32")
    assert skipped == 1, "out-of-pool slot not refused"
    expect_k = b.key_cache.copy()
    expect_v = b.value_cache.copy()
    for s in (0, 3):                            # only these two tokens are stored
        blk, off = divmod(int(b.slot_mapping[s]), b.block_size)
        expect_k[blk, :, off] = b.key[s]
        expect_v[blk, :, off] = b.value[s]
    assert np.array_equal(kc.view(np.uint8), expect_k.view(np.uint8)), "skip/refuse broke K"
    assert np.array_equal(vc.view(np.uint8), expect_v.view(np.uint8)), "skip/refuse broke V"


def pin_copy_blocks(orc):
    """Copy-on-write of shared blocks ([P2] 4.1, [P3] 2.2): every dst block equals its src in
    both caches afterwards, other blocks keep their bytes, ids outside the pool are refused."""
    b = W.build_batch("cow", [30, 50], num_heads=4, num_kv_heads=2, head_dim=64, block_size=8,
                      dtype="bf16", seed=W.BASE_SEED + 702, fill="zero", pool_factor=3.0)
    rng = np.random.default_rng(3)
    kc = W.encode(rng.standard_normal(b.key_cache.shape).astype(np.float32), "bf16")
    vc = W.encode(rng.standard_normal(b.value_cache.shape).astype(np.float32), "bf16")
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[0, 5], [3, 1], [7, 2], [0, 9]], np.int64)
    assert orc.copy_blocks(kc, vc, pairs, "bf16") == 0
    for src, dst in pairs:
        assert np.array_equal(kc[dst], k0[src]) and np.array_equal(vc[dst], v0[src])
    dsts = set(pairs[:, 1].tolist())
    for blk in range(kc.shape[0]):
        if blk not in dsts:
            assert np.array_equal(kc[blk], k0[blk]) and np.array_equal(vc[blk], v0[blk])
    bad = np.array([[0, kc.shape[0]], [-1, 4]], np.int64)
    k1 = kc.copy()
    assert orc.copy_blocks(kc, vc, bad, "bf16") == 2
    assert np.array_equal(kc, k1)


def pin_swap_blocks(orc):
    """Block-level swap ([P4] 2.3.2): blocks copied to a second pool equal their sources and
    nothing else there changes; a sequence swapped out, its device blocks overwritten, and
    swapped back into other free blocks (table updated) decodes to the same bits; ids outside
    either pool are refused."""
    b = W.build_batch("swap", [30, 50, 17], num_heads=8, num_kv_heads=2, head_dim=64,
                      block_size=8, dtype="bf16", seed=W.BASE_SEED + 705, pool_factor=3.0)
    orc.reshape_and_cache(b.key, b.value, b.key_cache, b.value_cache, b.slot_mapping, b.dtype)
    kc, vc = b.key_cache, b.value_cache
    nb = kc.shape[0]
    rng = np.random.default_rng(11)
    nh = nb + 16  # host pool larger than the device pool: every id below stays inside both
    hk = W.encode(rng.standard_normal((nh,) + kc.shape[1:]).astype(np.float32), "bf16")
    hv = W.encode(rng.standard_normal((nh,) + kc.shape[1:]).astype(np.float32), "bf16")
    before = orc.decode(b.query, kc, vc, b.block_tables, b.context_lens, b.scale, b.dtype)

    s = 1
    nblk = -(-int(b.context_lens[s]) // b.block_size)
    dev_ids = b.block_tables[s, :nblk].astype(np.int64)
    host_ids = rng.permutation(nb)[:nblk].astype(np.int64)  # below nb
    hk0, hv0 = hk.copy(), hv.copy()
    out_pairs = np.stack([dev_ids, host_ids], 1)
    assert orc.swap_blocks(kc, vc, hk, hv, out_pairs, "bf16") == 0
    for src, dst in out_pairs:
        assert np.array_equal(hk[dst], kc[src]) and np.array_equal(hv[dst], vc[src])
    for blk in set(range(nh)) - set(host_ids.tolist()):
        assert np.array_equal(hk[blk], hk0[blk]) and np.array_equal(hv[blk], hv0[blk])

    # the device blocks are reused by someone else; the sequence comes back elsewhere
    kc[dev_ids] = W.encode(np.full(kc[dev_ids].shape, np.nan, np.float32), "bf16")
    vc[dev_ids] = W.encode(np.full(vc[dev_ids].shape, np.nan, np.float32), "bf16")
    used = set()
    for q in range(b.num_seqs):
        used |= set(b.block_tables[q, :-(-int(b.context_lens[q]) // b.block_size)].tolist())
    free = np.array(sorted(set(range(nb)) - used), np.int64)
    new_ids = rng.permutation(free)[:nblk]
    assert orc.swap_blocks(hk, hv, kc, vc, np.stack([host_ids, new_ids], 1), "bf16") == 0
    tables = b.block_tables.copy()
    tables[s, :nblk] = new_ids
    after = orc.decode(b.query, kc, vc, tables, b.context_lens, b.scale, b.dtype)
    assert np.array_equal(after, before)

    k1, h1 = kc.copy(), hk.copy()
    bad_out = np.array([[0, nh], [nb, 0], [-1, 3]], np.int64)
    assert orc.swap_blocks(kc, vc, hk, hv, bad_out, "bf16") == 3
    assert np.array_equal(hk, h1) and np.array_equal(kc, k1)


def _torch_fp8_values():
    """The 256 E4M3 code values from torch's float8_e4m3fn type (a library decoder)."""
    import torch
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def pin_fp8_codec(orc):
    """FP8 E4M3 ([P2] 4.3 lists the format): the oracle's decoder agrees with torch's
    float8_e4m3fn on all 256 codes; its encoder agrees with torch's round-to-nearest-even cast
    on every finite bf16 value divided by several scales wherever torch's cast stays finite,
    saturates to +-448 beyond, keeps NaN as 0x7f, and decodes back to the same value."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = _torch_fp8_values()
    got = orc.fp8_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert got[0x7e] == 448.0 and got[0x08] == 2.0 ** -6 and got[0x01] == 2.0 ** -9
    assert np.all(np.diff(got[:0x7f]) > 0)  # codes 0..0x7e increase strictly
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32)
    bits = bits[np.isfinite(vals)]
    for scale in (1.0, 0.0078125, 0.37, 3.0):
        enc = orc.fp8_encode(bits, "bf16", scale)
        q = torch.from_numpy((bits.astype(np.uint32) << 16).view(np.float32)) / scale
        tq = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        inside = np.abs(q.numpy()) <= 464.0  # torch's cast is finite here
        assert np.array_equal(enc[inside], tq[inside]), scale
        big = ~inside
        assert np.all((enc[big] & 0x7f) == 0x7e)
        assert np.array_equal(enc[big] >> 7, (q.numpy()[big] < 0).astype(np.uint8))
    nan_bf16 = np.array([0x7fc0, 0xffc0], np.uint16)
    assert np.all(orc.fp8_encode(nan_bf16, "bf16", 1.0) == 0x7f)
    roundtrip = orc.fp8_encode(got[fin].astype(np.float32), "f32", 1.0)
    assert np.array_equal(orc.fp8_decode(roundtrip), got[fin])


def pin_fp8_cache(orc):
    """FP8 cache write and attention: each written slot holds the codes of its row divided by
    its kv head's scale, untouched and padding slots keep their bytes; the attention over an FP8
    cache equals long-double brute force over the decoded values times the per-head scales
    (keys and values scaled differently)."""
    b = W.build_batch("fp8", [1, 15, 16, 37, 60], num_heads=8, num_kv_heads=2, head_dim=64,
                      block_size=8, dtype="bf16", seed=W.BASE_SEED + 706, fill="zero",
                      keep_logical=True)
    nb, hkv, bs, d = b.key_cache.shape
    ks = np.array([0.011, 0.023], np.float32)
    vs = np.array([0.017, 0.0041], np.float32)
    kc = np.zeros((nb, hkv, bs, d), np.uint8)
    vc = np.zeros((nb, hkv, bs, d), np.uint8)
    # every token of every sequence through the write path
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        t = np.arange(L)
        slots = b.block_tables[s, t // bs].astype(np.int64) * bs + t % bs
        k_rows = np.ascontiguousarray(b.logical_key[s][:L])  # [L, Hkv, D]
        v_rows = np.ascontiguousarray(b.logical_value[s][:L])
        assert orc.reshape_and_cache_fp8(k_rows, v_rows, "bf16", kc, vc, slots, ks, vs) == 0
        for i in range(L):
            blk, off = slots[i] // bs, slots[i] % bs
            for h in range(hkv):
                assert np.array_equal(kc[blk, h, off], orc.fp8_encode(k_rows[i, h], "bf16", ks[h]))
                assert np.array_equal(vc[blk, h, off], orc.fp8_encode(v_rows[i, h], "bf16", vs[h]))
    k1, v1 = kc.copy(), vc.copy()
    pad = np.array([-1, nb * bs + 3], np.int64)
    rows = np.ones((2, hkv, d), np.uint16) * 0x3f80
    assert orc.reshape_and_cache_fp8(rows, rows, "bf16", kc, vc, pad, ks, vs) == 1
    assert np.array_equal(kc, k1) and np.array_equal(vc, v1)

    got = orc.decode(b.query, kc, vc, b.block_tables, b.context_lens, b.scale, "fp8",
                     q_dtype="bf16", k_scale=ks, v_scale=vs)
    table = _torch_fp8_values()
    q = W.decode_to_f64(b.query, "bf16").astype(np.longdouble)
    group = b.num_heads // hkv
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        t = np.arange(L)
        blk, off = b.block_tables[s, t // bs], t % bs
        for h in range(b.num_heads):
            g = h // group
            K = table[kc[blk, g, off]].astype(np.longdouble) * np.longdouble(ks[g])
            V = table[vc[blk, g, off]].astype(np.longdouble) * np.longdouble(vs[g])
            z = np.longdouble(b.scale) * (K @ q[s, h])
            w = np.exp(z - z.max())
            ref = (w @ V) / w.sum()
            assert np.allclose(got[s, h], ref.astype(np.float64), rtol=1e-12, atol=1e-15), (s, h)


def pin_prefill(orc):
    """Causal prefill ([P2] 4.2: requests join the batch with their prompt): every new token's
    row equals the decode oracle's attention of that query over the context positions 0 .. p
    (bit for bit: the same sum), torch's float64 scaled_dot_product_attention with a causal mask
    on the contiguous K/V agrees, and a 1-token chunk is exactly the decode step."""
    import torch
    b = W.build_prefill_batch("prefill", [5, 40, 17, 64, 9], [5, 13, 1, 30, 0], num_heads=8,
                              num_kv_heads=2, head_dim=64, block_size=8, dtype="bf16",
                              seed=W.BASE_SEED + 707, keep_logical=True)
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    assert orc.reshape_and_cache(b.key, b.value, kc, vc, b.slot_mapping, b.dtype) == 0
    got = orc.prefill(b.query, kc, vc, b.block_tables, b.context_lens, b.query_start, b.scale, b.dtype)
    qs = b.query_start
    group = b.num_heads // b.num_kv_heads
    for s in range(b.num_seqs):
        L, q0, q1 = int(b.context_lens[s]), int(qs[s]), int(qs[s + 1])
        for j in range(q1 - q0):
            p = L - (q1 - q0) + j
            one = orc.decode(b.query[q0 + j][None], kc, vc, b.block_tables[s][None],
                             np.array([p + 1], np.int32), b.scale, b.dtype)
            assert np.array_equal(got[q0 + j], one[0]), (s, j)
        if q1 == q0:
            continue
        K = torch.from_numpy(W.decode_to_f64(b.logical_key[s][:L], "bf16")).permute(1, 0, 2)
        V = torch.from_numpy(W.decode_to_f64(b.logical_value[s][:L], "bf16")).permute(1, 0, 2)
        Q = torch.from_numpy(W.decode_to_f64(b.query[q0:q1], "bf16")).permute(1, 0, 2)
        K = K.repeat_interleave(group, dim=0)
        V = V.repeat_interleave(group, dim=0)
        pos = torch.arange(L - (q1 - q0), L)[:, None]
        mask = torch.arange(L)[None, :] <= pos
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask,
                                                               scale=b.scale)
        assert np.allclose(got[q0:q1], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-14)
    last = orc.decode(b.query[qs[2]:qs[3]], kc, vc, b.block_tables[2:3], b.context_lens[2:3],
                      b.scale, b.dtype)
    assert np.array_equal(got[qs[2]:qs[3]], last)


def pin_shared_prefix(orc):
    """Sequences sharing prefix blocks read the same bytes: the paged result over the shared
    pool equals brute force on each member's own logical stream."""
    b = W.shared_prefix(num_groups=2, prefix_len=64, suffix_range=(16, 40), keep_logical=True)
    out, _, _ = _step(orc, b)
    err = _rel_err(out, brute_force(b).astype(np.float64))
    assert err < REL_TOL_F64, f"shared prefix rel err {err:.3e}"


def pin_split_merge(orc):
    """Split-context partitions merged with the log-sum-exp rule reproduce the unsplit
    result; empty partitions are neutral."""
    b = W.build_batch("split", [1, 20, 64, 100], num_heads=8, num_kv_heads=2, head_dim=128,
                      block_size=16, dtype="bf16", seed=W.BASE_SEED + 703)
    full, kc, vc = _step(orc, b)
    for bounds in ([0, 16, 48, 10 ** 6], [0, 1, 2, 3, 99, 10 ** 6], [0, 64, 64, 200, 10 ** 6]):
        parts = [orc.decode_range(b.query, kc, vc, b.block_tables, b.context_lens, b.scale,
                                  "bf16", lo, hi) for lo, hi in zip(bounds[:-1], bounds[1:])]
        for s in range(b.num_seqs):
            for h in range(b.num_heads):
                o = np.stack([p[0][s, h] for p in parts])
                m = np.array([p[1][s, h] for p in parts])
                l = np.array([p[2][s, h] for p in parts])
                merged = orc.lse_combine(o, m, l)
                assert _rel_err(merged, full[s, h]) < REL_TOL_F64, f"merge {bounds} s{s} h{h}"


def pin_zero_context(orc):
    """A sequence with no context gives a zero row; its neighbours are unaffected."""
    b = W.build_batch("zero", [0, 5, 0, 9], num_heads=4, num_kv_heads=1, head_dim=64,
                      block_size=8, dtype="f32", seed=W.BASE_SEED + 704, keep_logical=True)
    out, _, _ = _step(orc, b)
    assert np.all(out[0] == 0) and np.all(out[2] == 0), "empty context not zero"
    ref = brute_force(b).astype(np.float64)
    assert _rel_err(out[1], ref[1]) < REL_TOL_F64 and _rel_err(out[3], ref[3]) < REL_TOL_F64


ALL_PINS = [
    pin_brute_force, pin_torch_sdpa, pin_closed_forms, pin_decimal_example,
    pin_placement_invariance, pin_unread_table_entries, pin_cache_write, pin_copy_blocks,
    pin_swap_blocks, pin_fp8_codec, pin_fp8_cache, pin_prefill, pin_shared_prefix, pin_split_merge, pin_zero_context,
]
