"""Seeded synthetic inputs for paged KV-cache decode steps.

This module only *builds inputs*: the logical K/V stream of every sequence, the physical block
pool it is laid into, block tables, context lengths, the new tokens of the step with their
slots, copy-on-write block pairs and the queries.  It holds none of the attention arithmetic.
Both the CUDA path and the CPU oracle receive the very same bytes from it.

Shapes follow the library's conventions:
  query        [S, Hq, D]
  key_cache    [NB, Hkv, bs, D]   (value_cache alike): the pool *before* the step's writes
  key, value   [T, Hkv, D]        tokens written this step, at slot_mapping [T] (int64)
  block_tables [S, max_blocks]    int32, -1 past a sequence's last block (never read)
  context_lens [S]                int32, counting the token written this step
  block_mapping [N, 2]            int64 (src, dst) copies that precede the step's writes
Element storage: "f32" -> float32, "bf16" -> uint16 bit patterns, "f16" -> float16.

Every value is drawn from numpy's PCG64 with a documented seed (base seed 42700 + config
number), N(0, 1) in float32 and rounded to nearest-even when stored as bf16.  Each sequence's
values come from their own generator so a batch can be built in pieces.  Pool slots that no
sequence uses, and slots past a sequence's context, are filled with NaN (``fill="nan"``) so that
any read of them would poison the result.

Sources for the structure (vLLM tutorials, by page and section): [P2] "vLLM core features:
PagedAttention, Continuous Batching, quantization support, distributed inference" 4.1 (block
table, one mapping appended per generated token, shared physical blocks); [P3] "Core inference
engine (part 1): vLLM architecture, PagedAttention principle, Continuous Batching mechanism" 2.2
(page of 16 tokens; a service with mean request length 200 against a 2048 preallocation; page
size 8 vs 32); [P4] "vLLM core architecture: model loading, PagedAttention principle, KV cache
management" 2.2.1 (logical block, physical block, block table; block size 16 by default, 8 for
short texts, 32 for long ones).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BASE_SEED = 42700
STORAGE = {"f32": np.float32, "bf16": np.uint16, "f16": np.float16}
NAN_BITS = {"bf16": np.uint16(0x7FC0), "f16": np.float16(np.nan), "f32": np.float32(np.nan)}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns the uint16 patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def encode(x: np.ndarray, dtype: str) -> np.ndarray:
    """Store float32 values in the given element type."""
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    if dtype == "f16":
        return np.asarray(x, dtype=np.float32).astype(np.float16)
    return np.asarray(x, dtype=np.float32)


def decode_to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Widen stored elements to float64 (exact)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x).astype(np.float64)


def _normal(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    return encode(rng.standard_normal(shape, dtype=np.float32), dtype)


@dataclass
class PagedBatch:
    """One decode step's inputs (host numpy arrays)."""

    name: str
    dtype: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    query: np.ndarray
    key_cache: np.ndarray
    value_cache: np.ndarray
    key: np.ndarray
    value: np.ndarray
    slot_mapping: np.ndarray
    block_tables: np.ndarray
    context_lens: np.ndarray
    block_mapping: np.ndarray | None = None
    # Per-sequence logical K/V streams after the step ([L, Hkv, D] each), kept only on request.
    logical_key: list | None = None
    logical_value: list | None = None
    meta: dict = field(default_factory=dict)
    # Prefill steps: the new tokens of sequence s are query rows query_start[s] ..
    # query_start[s+1]-1 (and key/value/slot_mapping rows alike), the last positions of its
    # context.  None for decode steps (one new token per sequence).
    query_start: np.ndarray | None = None

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_blocks(self) -> int:
        return int(self.key_cache.shape[0])

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def attended_tokens(self) -> int:
        return int(np.maximum(self.context_lens, 0).sum())


def _fill_pool(shape, dtype: str, fill: str) -> np.ndarray:
    if fill == "nan":
        return np.full(shape, NAN_BITS[dtype], dtype=STORAGE[dtype])
    if fill == "zero":
        return np.zeros(shape, dtype=STORAGE[dtype])
    raise ValueError(fill)


def _assign_blocks(context_lens, block_size: int, num_blocks: int | None, pool_factor: float,
                   rng: np.random.Generator, max_blocks: int | None):
    """Give each sequence ceil(L/bs) distinct physical blocks from a shuffled pool."""
    lens = np.asarray(context_lens, dtype=np.int64)
    nblk = (lens + block_size - 1) // block_size
    total = int(nblk.sum())
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(pool_factor * total)))
    if total > num_blocks:
        raise ValueError(f"pool of {num_blocks} blocks cannot hold {total}")
    if max_blocks is None:
        max_blocks = max(1, int(nblk.max()) if len(nblk) else 1)
    perm = rng.permutation(num_blocks)[:total].astype(np.int32)
    tables = np.full((len(lens), max_blocks), -1, dtype=np.int32)
    start = 0
    for s, n in enumerate(nblk):
        tables[s, :n] = perm[start:start + n]
        start += n
    return tables, num_blocks


def _place(pool: np.ndarray, table_row: np.ndarray, first: int, rows: np.ndarray, block_size: int):
    """Lay logical rows [first, first+len(rows)) of one sequence into its physical blocks."""
    if len(rows) == 0:
        return
    t = np.arange(first, first + len(rows))
    pool[table_row[t // block_size], :, t % block_size, :] = rows


def build_batch(name: str, context_lens, *, num_heads: int, num_kv_heads: int, head_dim: int,
                block_size: int, dtype: str, seed: int, num_blocks: int | None = None,
                pool_factor: float = 1.25, max_blocks: int | None = None, fill: str = "nan",
                keep_logical: bool = False, perm_salt: int = 0) -> PagedBatch:
    """Generic decode step: every sequence owns its blocks; its last token is written this step.

    Values of sequence s come from PCG64([seed, 1, s]); the block permutation from
    PCG64([seed, 3, perm_salt]); queries from PCG64([seed, 2]).  Changing block_size or
    perm_salt therefore changes the placement only, never the logical values.
    """
    lens = np.asarray(context_lens, dtype=np.int32)
    S = len(lens)
    tables, nb = _assign_blocks(lens, block_size, num_blocks, pool_factor,
                                np.random.default_rng([seed, 3, perm_salt]), max_blocks)
    kc = _fill_pool((nb, num_kv_heads, block_size, head_dim), dtype, fill)
    vc = _fill_pool((nb, num_kv_heads, block_size, head_dim), dtype, fill)
    key = np.zeros((S, num_kv_heads, head_dim), dtype=STORAGE[dtype])
    value = np.zeros((S, num_kv_heads, head_dim), dtype=STORAGE[dtype])
    slots = np.full(S, -1, dtype=np.int64)
    lk, lv = ([], []) if keep_logical else (None, None)
    for s in range(S):
        L = int(lens[s])
        rng = np.random.default_rng([seed, 1, s])
        ks = _normal(rng, (L, num_kv_heads, head_dim), dtype)
        vs = _normal(rng, (L, num_kv_heads, head_dim), dtype)
        if L > 0:
            _place(kc, tables[s], 0, ks[:L - 1], block_size)
            _place(vc, tables[s], 0, vs[:L - 1], block_size)
            key[s], value[s] = ks[L - 1], vs[L - 1]
            slots[s] = int(tables[s, (L - 1) // block_size]) * block_size + (L - 1) % block_size
        if keep_logical:
            lk.append(ks)
            lv.append(vs)
    query = _normal(np.random.default_rng([seed, 2]), (S, num_heads, head_dim), dtype)
    return PagedBatch(name=name, dtype=dtype, num_heads=num_heads, num_kv_heads=num_kv_heads,
                      head_dim=head_dim, block_size=block_size, scale=1.0 / math.sqrt(head_dim),
                      query=query, key_cache=kc, value_cache=vc, key=key, value=value,
                      slot_mapping=slots, block_tables=tables, context_lens=lens,
                      logical_key=lk, logical_value=lv,
                      meta={"seed": seed, "perm_salt": perm_salt, "fill": fill})


def build_prefill_batch(name: str, context_lens, q_lens, *, num_heads: int, num_kv_heads: int,
                        head_dim: int, block_size: int, dtype: str, seed: int,
                        pool_factor: float = 1.25, max_blocks: int | None = None,
                        fill: str = "nan", keep_logical: bool = False) -> PagedBatch:
    """A step in which sequence s brings q_lens[s] new tokens (a prompt chunk; 1 = a decode
    token): positions context_lens[s] - q_lens[s] .. context_lens[s] - 1.  The pool holds each
    sequence's earlier tokens; the new tokens' rows and slots are the step's write, and their
    query rows are concatenated in sequence order.  Values as in build_batch."""
    lens = np.asarray(context_lens, dtype=np.int32)
    ql = np.asarray(q_lens, dtype=np.int32)
    if np.any(ql < 0) or np.any(ql > lens):
        raise ValueError("0 <= q_len <= context_len")
    S = len(lens)
    tables, nb = _assign_blocks(lens, block_size, None, pool_factor,
                                np.random.default_rng([seed, 3, 0]), max_blocks)
    kc = _fill_pool((nb, num_kv_heads, block_size, head_dim), dtype, fill)
    vc = _fill_pool((nb, num_kv_heads, block_size, head_dim), dtype, fill)
    keys, values, slots = [], [], []
    lk, lv = ([], []) if keep_logical else (None, None)
    for s in range(S):
        L, q = int(lens[s]), int(ql[s])
        rng = np.random.default_rng([seed, 1, s])
        ks = _normal(rng, (L, num_kv_heads, head_dim), dtype)
        vs = _normal(rng, (L, num_kv_heads, head_dim), dtype)
        _place(kc, tables[s], 0, ks[:L - q], block_size)
        _place(vc, tables[s], 0, vs[:L - q], block_size)
        t = np.arange(L - q, L)
        keys.append(ks[L - q:])
        values.append(vs[L - q:])
        slots.append(tables[s, t // block_size].astype(np.int64) * block_size + t % block_size)
        if keep_logical:
            lk.append(ks)
            lv.append(vs)
    total = int(ql.sum())
    query = _normal(np.random.default_rng([seed, 2]), (total, num_heads, head_dim), dtype)
    qs = np.zeros(S + 1, dtype=np.int32)
    qs[1:] = np.cumsum(ql)
    return PagedBatch(name=name, dtype=dtype, num_heads=num_heads, num_kv_heads=num_kv_heads,
                      head_dim=head_dim, block_size=block_size, scale=1.0 / math.sqrt(head_dim),
                      query=query, key_cache=kc, value_cache=vc,
                      key=np.concatenate(keys) if keys else np.zeros((0, num_kv_heads, head_dim), STORAGE[dtype]),
                      value=np.concatenate(values) if values else np.zeros((0, num_kv_heads, head_dim), STORAGE[dtype]),
                      slot_mapping=np.concatenate(slots) if slots else np.zeros(0, np.int64),
                      block_tables=tables, context_lens=lens, logical_key=lk,
                      logical_value=lv, meta={"seed": seed, "fill": fill}, query_start=qs)


def chunked_prefill(num_seqs: int = 8, chunk: int = 256, max_context: int = 2048,
                    seed: int = BASE_SEED + 6) -> PagedBatch:
    """Chunked prefill on Llama-3-8B shapes (32/8 heads, head_dim 128, bf16, block_size 16):
    each sequence brings a prompt chunk of `chunk` tokens on top of an earlier prefix of
    U[0, max_context - chunk] tokens (rounded to whole chunks)."""
    rng = np.random.default_rng([seed, 0])
    prefix = rng.integers(0, (max_context - chunk) // chunk + 1, num_seqs) * chunk
    lens = (prefix + chunk).astype(np.int32)
    return build_prefill_batch("chunked_prefill", lens, np.full(num_seqs, chunk, np.int32),
                               num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                               dtype="bf16", seed=seed)


# ----------------------------------------------------------------------------------------------
# The five workloads.  Full sizes by default; smaller variants (fewer sequences, shorter
# contexts) keep the same structure for tests the CPU oracle must finish in seconds.
# ----------------------------------------------------------------------------------------------

def tiny_fp32(fill: str = "nan", keep_logical: bool = True) -> PagedBatch:
    """4 sequences, contexts {1, 15, 16, 37}, 4 query heads = 4 KV heads, head_dim 64, fp32,
    block_size 16, a pool of 32 blocks assigned by seeded permutation, scale 1/8."""
    return build_batch("tiny_fp32", [1, 15, 16, 37], num_heads=4, num_kv_heads=4, head_dim=64,
                       block_size=16, dtype="f32", seed=BASE_SEED + 1, num_blocks=32, fill=fill,
                       keep_logical=keep_logical)


def llama3_8b_decode(num_seqs: int = 64, min_len: int = 128, max_len: int = 2048,
                     block_size: int = 16, dtype: str = "bf16", fill: str = "nan",
                     keep_logical: bool = False, seed: int = BASE_SEED + 2) -> PagedBatch:
    """Llama-3-8B-shaped decode step: 32 query heads / 8 KV heads, head_dim 128, bf16,
    block_size 16, context lengths uniform in [min_len, max_len]; the pool holds max_len tokens
    per sequence (8192 blocks at full size) and is assigned by random permutation."""
    rng = np.random.default_rng([seed, 0])
    lens = rng.integers(min_len, max_len + 1, size=num_seqs).astype(np.int32)
    nb = num_seqs * ((max_len + block_size - 1) // block_size)
    return build_batch("llama3_8b_decode", lens, num_heads=32, num_kv_heads=8, head_dim=128,
                       block_size=block_size, dtype=dtype, seed=seed, num_blocks=nb,
                       max_blocks=(max_len + block_size - 1) // block_size, fill=fill,
                       keep_logical=keep_logical)


def short_chat_lens(num_seqs: int = 256, median: float = 200.0, sigma: float = 1.0,
                    max_len: int = 2048, seed: int = BASE_SEED + 3) -> np.ndarray:
    """Lognormal context lengths (median 200, sigma 1), rounded and clipped to [1, max_len]."""
    rng = np.random.default_rng([seed, 0])
    x = median * np.exp(sigma * rng.standard_normal(num_seqs))
    return np.clip(np.rint(x), 1, max_len).astype(np.int32)


def short_chat(block_size: int, num_seqs: int = 256, max_len: int = 2048, fill: str = "nan",
               keep_logical: bool = False, seed: int = BASE_SEED + 3) -> PagedBatch:
    """Block-size sweep case: identical logical K/V for block_size 8, 16 and 32; independent
    shuffled pools (1.25x the blocks needed) per block size."""
    lens = short_chat_lens(num_seqs=num_seqs, max_len=max_len, seed=seed)
    return build_batch(f"short_chat_bs{block_size}", lens, num_heads=32, num_kv_heads=8,
                       head_dim=128, block_size=block_size, dtype="bf16", seed=seed,
                       max_blocks=(max_len + block_size - 1) // block_size, fill=fill,
                       keep_logical=keep_logical, perm_salt=block_size)


def long_mixed_lens(num_long: int = 16, long_range=(8192, 32768), num_short: int = 240,
                    short_range=(16, 1024), seed: int = BASE_SEED + 5) -> np.ndarray:
    """16 long contexts U[8192, 32768] and 240 short ones U[16, 1024], in shuffled order."""
    rng = np.random.default_rng([seed, 0])
    lens = np.concatenate([rng.integers(long_range[0], long_range[1] + 1, size=num_long),
                           rng.integers(short_range[0], short_range[1] + 1, size=num_short)])
    return lens[rng.permutation(len(lens))].astype(np.int32)


def long_mixed(num_long: int = 16, long_range=(8192, 32768), num_short: int = 240,
               short_range=(16, 1024), fill: str = "nan", keep_logical: bool = False,
               seed: int = BASE_SEED + 5) -> PagedBatch:
    """Mixed continuous-batching step with long contexts: GQA 32/8, head_dim 128, bf16,
    block_size 16, shuffled pool of 1.25x the blocks needed, block tables wide enough for the
    longest allowed context."""
    lens = long_mixed_lens(num_long, long_range, num_short, short_range, seed)
    return build_batch("long_mixed", lens, num_heads=32, num_kv_heads=8, head_dim=128,
                       block_size=16, dtype="bf16", seed=seed,
                       max_blocks=(long_range[1] + 15) // 16, fill=fill,
                       keep_logical=keep_logical)


def shared_prefix(num_groups: int = 32, group_size: int = 4, prefix_len: int = 1024,
                  suffix_range=(16, 512), block_size: int = 16, fill: str = "nan",
                  keep_logical: bool = False, seed: int = BASE_SEED + 4) -> PagedBatch:
    """Parallel-sampling batch sharing one system prompt.

    All sequences share a prefix of prefix_len tokens stored once (prefix_len / block_size
    physical blocks).  Each group also shares a prompt tail of p_g ~ U[1, block_size-1] tokens
    held in one group block.  Member 0 of a group keeps that block; members 1.. get a
    copy-on-write copy of it (block_mapping), after which the step writes each member's own
    tokens into the rest of its tail block.  A member's context is prefix_len + u with
    u ~ U[suffix_range] counting the p_g tail tokens; its tokens after the tail block are its
    own and already in the pool; its last token is written this step.
    """
    if prefix_len % block_size:
        raise ValueError("prefix must fill whole blocks")
    Hq, Hkv, D = 32, 8, 128
    dtype = "bf16"
    S = num_groups * group_size
    rng = np.random.default_rng([seed, 0])
    tails = rng.integers(1, block_size, size=num_groups)               # p_g
    u = rng.integers(suffix_range[0], suffix_range[1] + 1, size=S)     # suffix incl. the tail
    lens = (prefix_len + u).astype(np.int32)
    n_prefix = prefix_len // block_size
    nblk = (lens.astype(np.int64) + block_size - 1) // block_size
    own = nblk - n_prefix - 1                                           # blocks after the tail
    needed = n_prefix + S + int(own.sum())                              # prefix + tail copies + own
    nb = int(math.ceil(1.25 * needed))
    perm = np.random.default_rng([seed, 3]).permutation(nb).astype(np.int32)
    max_blocks = (prefix_len + suffix_range[1] + block_size - 1) // block_size
    tables = np.full((S, max_blocks), -1, dtype=np.int32)
    prefix_blocks = perm[:n_prefix]
    tail_blocks = perm[n_prefix:n_prefix + S].reshape(num_groups, group_size)
    cursor = n_prefix + S
    for s in range(S):
        tables[s, :n_prefix] = prefix_blocks
        tables[s, n_prefix] = tail_blocks[s // group_size, s % group_size]
        tables[s, n_prefix + 1:nblk[s]] = perm[cursor:cursor + own[s]]
        cursor += own[s]
    kc = _fill_pool((nb, Hkv, block_size, D), dtype, fill)
    vc = _fill_pool((nb, Hkv, block_size, D), dtype, fill)
    prng = np.random.default_rng([seed, 10])
    pk = _normal(prng, (prefix_len, Hkv, D), dtype)
    pv = _normal(prng, (prefix_len, Hkv, D), dtype)
    _place(kc, tables[0], 0, pk, block_size)
    _place(vc, tables[0], 0, pv, block_size)
    mapping = []
    writes_k, writes_v, writes_slot = [], [], []
    lk, lv = ([], []) if keep_logical else (None, None)
    group_tail = {}
    for g in range(num_groups):
        trng = np.random.default_rng([seed, 11, g])
        tk = _normal(trng, (int(tails[g]), Hkv, D), dtype)
        tv = _normal(trng, (int(tails[g]), Hkv, D), dtype)
        group_tail[g] = (tk, tv)
        # the shared tail lives in member 0's block; members 1.. copy it before writing
        _place(kc, tables[g * group_size], prefix_len, tk, block_size)
        _place(vc, tables[g * group_size], prefix_len, tv, block_size)
        for i in range(1, group_size):
            mapping.append((int(tail_blocks[g, 0]), int(tail_blocks[g, i])))
    tail_end = prefix_len + block_size                                  # end of the tail block
    for s in range(S):
        g = s // group_size
        L = int(lens[s])
        p = int(tails[g])
        srng = np.random.default_rng([seed, 1, s])
        n_own = L - prefix_len - p
        ok = _normal(srng, (n_own, Hkv, D), dtype)
        ov = _normal(srng, (n_own, Hkv, D), dtype)
        first_own = prefix_len + p
        # positions [first_own, tail_end) sit in the (possibly copied) tail block: written this
        # step after the copies; positions from tail_end on are already in the member's blocks,
        # except the last token, which is written this step.
        n_in_tail = min(tail_end, L) - first_own
        after = ok[n_in_tail:max(n_in_tail, n_own - 1)]
        _place(kc, tables[s], tail_end, after, block_size)
        _place(vc, tables[s], tail_end, ov[n_in_tail:max(n_in_tail, n_own - 1)], block_size)
        positions = list(range(first_own, first_own + n_in_tail))
        if L - 1 not in positions:
            positions.append(L - 1)
        for t in positions:
            j = t - first_own
            writes_k.append(ok[j])
            writes_v.append(ov[j])
            writes_slot.append(int(tables[s, t // block_size]) * block_size + t % block_size)
        if keep_logical:
            tk, tv = group_tail[g]
            lk.append(np.concatenate([pk, tk, ok]))
            lv.append(np.concatenate([pv, tv, ov]))
    query = _normal(np.random.default_rng([seed, 2]), (S, Hq, D), dtype)
    return PagedBatch(name="shared_prefix", dtype=dtype, num_heads=Hq, num_kv_heads=Hkv,
                      head_dim=D, block_size=block_size, scale=1.0 / math.sqrt(D), query=query,
                      key_cache=kc, value_cache=vc, key=np.stack(writes_k),
                      value=np.stack(writes_v), slot_mapping=np.asarray(writes_slot, np.int64),
                      block_tables=tables, context_lens=lens,
                      block_mapping=np.asarray(mapping, dtype=np.int64).reshape(-1, 2),
                      logical_key=lk, logical_value=lv,
                      meta={"seed": seed, "tails": tails.tolist(), "prefix_len": prefix_len,
                            "group_size": group_size, "fill": fill})


def shared_groups(b: PagedBatch):
    """The batch's prefix sharing for pa_decode_shared_prefix: (group_start [num_groups + 1],
    prefix_lens [num_seqs]) int32.  The shared-prefix batch is one group whose members share
    its whole-block system prompt; any other batch is one group per sequence sharing nothing."""
    S = b.num_seqs
    if "prefix_len" in b.meta:
        return (np.array([0, S], dtype=np.int32),
                np.full(S, int(b.meta["prefix_len"]), dtype=np.int32))
    return np.arange(S + 1, dtype=np.int32), np.zeros(S, dtype=np.int32)


def workload(name: str, **kw) -> PagedBatch:
    """Build a workload by name: tiny_fp32, llama3_8b_decode, short_chat_bs{8,16,32},
    shared_prefix, long_mixed."""
    if name == "tiny_fp32":
        return tiny_fp32(**kw)
    if name == "llama3_8b_decode":
        return llama3_8b_decode(**kw)
    if name.startswith("short_chat_bs"):
        return short_chat(int(name[len("short_chat_bs"):]), **kw)
    if name == "shared_prefix":
        return shared_prefix(**kw)
    if name == "long_mixed":
        return long_mixed(**kw)
    if name == "chunked_prefill":
        return chunked_prefill(**kw)
    raise KeyError(name)


def sub_batch(batch: PagedBatch, seqs) -> dict:
    """The decode inputs of a subset of sequences (same pool): for sampled oracle checks."""
    seqs = np.asarray(seqs, dtype=np.int64)
    return dict(query=batch.query[seqs], block_tables=batch.block_tables[seqs],
                context_lens=batch.context_lens[seqs])
