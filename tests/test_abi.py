"""The C-ABI library builds, loads and exports what include/pa.h declares; host-side argument
checks run before any CUDA call, so they are exercised here without a GPU."""
import ctypes
import re
import subprocess

import pytest

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import build as pa_build


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return pa.load()


def test_every_declared_function_is_exported(lib):
    declared = pa.header_functions()
    assert {"pa_reshape_and_cache", "pa_copy_blocks", "pa_decode", "pa_decode_ex"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIBRARY], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(pa_\w+)$", out, re.M))
    missing = [f for f in declared if f not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for f in declared:
        assert hasattr(lib, f)
    # nothing but the C ABI leaks out of the library
    assert not [s for s in re.findall(r"\sT\s(\S+)$", out, re.M) if not s.startswith("pa_")
                and not s.startswith("_init") and not s.startswith("_fini")]


# The boundary's calls as first proposed (name: what it does) and the exported calls that
# provide each; the argument changes are documented beside each declaration in include/pa.h.
PROPOSED_TO_PROVIDED = {
    "pa_reshape_and_cache": ["pa_reshape_and_cache"],
    "pa_decode": ["pa_decode"],
    # partition_size became num_workers + flags (the split is by bytes over warps, stream-K)
    "pa_decode_ex": ["pa_decode_ex"],
    # sized by sequences, heads, head_dim and warps instead of table width and partition size
    "pa_decode_workspace_bytes": ["pa_decode_workspace_bytes", "pa_decode_default_workers"],
    "pa_copy_blocks": ["pa_copy_blocks"],
    "pa_last_error": ["pa_last_error"],
    # gained a `clear` argument
    "pa_get_device_error": ["pa_get_device_error"],
    # freeing the library-owned workspaces
    "pa_shutdown": ["pa_release_workspaces"],
    # zero-filling a caller workspace before its first use
    "(workspace set-up)": ["pa_workspace_init"],
}


def test_every_proposed_call_is_provided(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIBRARY], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(pa_\w+)$", out, re.M))
    declared = set(pa.header_functions())
    for proposed, provided in PROPOSED_TO_PROVIDED.items():
        for name in provided:
            assert name in exported and name in declared, f"{proposed}: {name} not provided"


def test_version_matches_header(lib):
    with open(pa.HEADER) as f:
        v = int(re.search(r"#define PA_VERSION (\d+)", f.read()).group(1))
    assert pa.pa_version() == v


def test_workspace_bytes_layout(lib):
    # counters [S*Hkv] u32 | pair_meta [S*Hkv] int2 | part_ml [(S*Hkv+W)*G*2] f32 |
    # part_o [(S*Hkv+W)*G*D] f32, each region rounded up to 256 bytes
    def up(x):
        return (x + 255) // 256 * 256

    S, Hq, Hkv, D, W = 64, 32, 8, 128, 1184
    pairs, segs, G = S * Hkv, S * Hkv + W, Hq // Hkv
    expect = up(pairs * 4) + up(pairs * 8) + up(segs * G * 2 * 4) + up(segs * G * D * 4)
    assert pa.pa_decode_workspace_bytes(S, Hq, Hkv, D, W) == expect
    assert pa.pa_decode_workspace_bytes(S, 30, 8, D, W) == 0  # heads not a multiple
    assert pa.pa_decode_workspace_bytes(-1, Hq, Hkv, D, W) == 0


def _t(shape, dtype, data=0x10000, stride=None):
    d = pa.PaTensor()
    d.data = data
    d.dtype = dtype
    d.ndim = len(shape)
    if stride is None:
        stride, acc = [], 1
        for n in reversed(shape):
            stride.insert(0, acc)
            acc *= n
    for i, (n, s) in enumerate(zip(shape, stride)):
        d.shape[i] = n
        d.stride[i] = s
    return d


def _decode_args(S=4, Hq=8, Hkv=2, D=128, bs=16, NB=32, MB=4, dt=pa.PA_BF16, out_dt=None,
                 q_data=0x10000):
    return dict(out=_t([S, Hq, D], out_dt if out_dt is not None else dt),
                query=_t([S, Hq, D], dt, data=q_data),
                kc=_t([NB, Hkv, bs, D], dt), vc=_t([NB, Hkv, bs, D], dt),
                bt=_t([S, MB], pa.PA_I32), cl=_t([S], pa.PA_I32))


def _decode(lib, a, bs=16, hkv=2, flags=0, workers=0, scale=0.1):
    r = ctypes.byref
    return lib.pa_decode_ex(r(a["out"]), r(a["query"]), r(a["kc"]), r(a["vc"]), r(a["bt"]),
                            r(a["cl"]), scale, bs, hkv, workers, flags, None, 0, None)


@pytest.mark.parametrize("case,expect", [
    (dict(D=96), -4),                        # head_dim not built
    (dict(bs=64), -4),                       # block_size not built
    (dict(Hq=24, Hkv=2), -4),                # group of 12 not built
    (dict(Hq=7, Hkv=2), -2),                 # heads not a multiple of kv heads
    (dict(out_dt=pa.PA_F16), -3),            # out neither fp32 nor the cache type
    (dict(q_data=0x10008), -7),              # query misaligned
])
def test_decode_rejects_bad_arguments_before_cuda(lib, case, expect):
    kw = dict(case)
    a = _decode_args(**kw)
    assert _decode(lib, a, bs=kw.get("bs", 16), hkv=kw.get("Hkv", 2)) == expect
    assert pa.pa_last_error()


def test_decode_rejects_mismatches(lib):
    a = _decode_args()
    assert _decode(lib, a, bs=8) == -2          # block_size disagrees with the cache
    assert _decode(lib, a, hkv=4) == -2         # num_kv_heads disagrees with the cache
    assert _decode(lib, a, flags=0x80) == -1    # unknown flag
    assert _decode(lib, a, workers=-1) == -1
    assert _decode(lib, a, scale=float("nan")) == -1
    b = _decode_args()
    b["vc"] = _t([32, 2, 16, 128], pa.PA_F16)
    assert _decode(lib, b) == -3                 # caches of different types
    c = _decode_args()
    c["bt"] = _t([4, 4], pa.PA_I64)
    assert _decode(lib, c) == -3                 # block table must be int32
    d = _decode_args()
    d["kc"] = _t([32, 2, 16, 128], pa.PA_BF16, stride=[4096, 2048, 256, 1])
    d["vc"] = _t([32, 2, 16, 128], pa.PA_BF16, stride=[4096, 2048, 256, 1])
    assert _decode(lib, d) == -7                 # tile rows not contiguous
    e = _decode_args()
    e["cl"] = _t([3], pa.PA_I32)
    assert _decode(lib, e) == -2                 # one context length per sequence


def test_decode_rejects_a_step_too_large_for_the_work_split(lib):
    # 16 sequences x 2 kv heads x 2^31 - 16 positions: 2^32 chunks of 16 positions, past the
    # 2e9 a worker's 32-bit chunk count allows (each table alone is within its own bound)
    mb = (2**31 - 16) // 16
    a = _decode_args(S=16, Hq=4, Hkv=2, MB=mb)
    assert _decode(lib, a) == -2
    assert "too large" in pa.pa_last_error()
    ok = _decode_args(S=16, Hq=4, Hkv=2, MB=mb // 64)  # 2^26 chunks: passes this check
    assert _decode(lib, ok) != -2


def test_zero_sequences_is_a_no_op(lib):
    a = _decode_args(S=0)
    assert _decode(lib, a) == 0


def test_reshape_and_cache_rejects_bad_arguments(lib):
    r = ctypes.byref
    kc = _t([32, 2, 16, 128], pa.PA_BF16)
    vc = _t([32, 2, 16, 128], pa.PA_BF16)
    key = _t([5, 2, 128], pa.PA_BF16)
    val = _t([5, 2, 128], pa.PA_BF16)
    slots32 = _t([5], pa.PA_I32)
    assert lib.pa_reshape_and_cache(r(key), r(val), r(kc), r(vc), r(slots32), None) == -3
    slots = _t([4], pa.PA_I64)
    assert lib.pa_reshape_and_cache(r(key), r(val), r(kc), r(vc), r(slots), None) == -2
    key3 = _t([5, 3, 128], pa.PA_BF16)
    assert lib.pa_reshape_and_cache(r(key3), r(key3), r(kc), r(vc), r(_t([5], pa.PA_I64)), None) == -2
    empty = _t([0, 2, 128], pa.PA_BF16)
    assert lib.pa_reshape_and_cache(r(empty), r(empty), r(kc), r(vc), r(_t([0], pa.PA_I64)), None) == 0


def test_copy_blocks_rejects_bad_arguments(lib):
    r = ctypes.byref
    kc = _t([32, 2, 16, 128], pa.PA_BF16)
    vc = _t([32, 2, 16, 128], pa.PA_BF16)
    assert lib.pa_copy_blocks(r(kc), r(vc), r(_t([3, 3], pa.PA_I64)), None) == -2
    assert lib.pa_copy_blocks(r(kc), r(vc), r(_t([3, 2], pa.PA_I32)), None) == -3
    assert lib.pa_copy_blocks(r(kc), r(vc), r(_t([0, 2], pa.PA_I64)), None) == 0


def test_decode_step_checks_both_halves_first(lib):
    r = ctypes.byref
    a = _decode_args()
    key = _t([4, 2, 128], pa.PA_BF16)
    slots = _t([4], pa.PA_I64)

    def step(key=key, slots=slots, a=a, bs=16):
        return lib.pa_decode_step(r(key), r(key), r(a["kc"]), r(a["vc"]), r(slots), r(a["out"]),
                                  r(a["query"]), r(a["bt"]), r(a["cl"]), 0.1, bs, 2, None, 0, None)

    assert step(slots=_t([4], pa.PA_I32)) == -3        # write half: slots must be int64
    assert step(key=_t([4, 3, 128], pa.PA_BF16)) == -2  # write half: kv heads of the cache
    assert step(bs=8) == -2                             # decode half: block_size mismatch
    b = _decode_args(D=96)
    assert step(key=_t([4, 2, 96], pa.PA_BF16), a=b) == -4  # decode half: head_dim not built
    assert pa.pa_last_error()


def test_status_constants_match_header():
    with open(pa.HEADER) as f:
        text = f.read()
    for name, value in re.findall(r"\b(PA_ERR_[A-Z_]+)\s*=\s*(-\d+)", text):
        assert getattr(pa, name) == int(value), name


def _prefill_args(S=3, T=40, Hq=8, Hkv=2, D=128, bs=16, NB=32, MB=8, dt=pa.PA_BF16, out_dt=None,
                  q_data=0x10000, qs_len=None):
    return dict(out=_t([T, Hq, D], out_dt if out_dt is not None else dt),
                query=_t([T, Hq, D], dt, data=q_data),
                kc=_t([NB, Hkv, bs, D], dt), vc=_t([NB, Hkv, bs, D], dt),
                bt=_t([S, MB], pa.PA_I32), cl=_t([S], pa.PA_I32),
                qs=_t([qs_len if qs_len is not None else S + 1], pa.PA_I32))


def _prefill(lib, a, bs=16, hkv=2, scale=0.1):
    r = ctypes.byref
    return lib.pa_prefill(r(a["out"]), r(a["query"]), r(a["kc"]), r(a["vc"]), r(a["bt"]), r(a["cl"]),
                          r(a["qs"]), scale, bs, hkv, None)


@pytest.mark.parametrize("case,expect", [
    (dict(D=96), -4),                        # head_dim not built
    (dict(bs=64), -4),                       # block_size not built
    (dict(Hq=24, Hkv=2), -4),                # group of 12 not built
    (dict(Hq=7, Hkv=2), -2),                 # heads not a multiple of kv heads
    (dict(dt=pa.PA_F32), -4),                # prefill is built for 16-bit caches
    (dict(out_dt=pa.PA_F16), -3),            # out neither fp32 nor the cache type
    (dict(qs_len=3), -2),                    # query_start needs S + 1 entries
    (dict(q_data=0x10008), -7),              # query misaligned
])
def test_prefill_rejects_bad_arguments_before_cuda(lib, case, expect):
    kw = dict(case)
    a = _prefill_args(**kw)
    assert _prefill(lib, a, bs=kw.get("bs", 16), hkv=kw.get("Hkv", 2)) == expect
    assert pa.pa_last_error()


def test_prefill_rejects_mismatches(lib):
    a = _prefill_args()
    assert _prefill(lib, a, bs=8) == -2           # block_size disagrees with the cache
    assert _prefill(lib, a, hkv=4) == -2          # num_kv_heads disagrees with the cache
    assert _prefill(lib, a, scale=float("inf")) == -1
    b = _prefill_args()
    b["query"] = _t([40, 8, 128], pa.PA_F16)
    assert _prefill(lib, b) == -3                 # query of another type than the caches
    c = _prefill_args()
    c["qs"] = _t([4], pa.PA_I64)
    assert _prefill(lib, c) == -3                 # query_start must be int32
    d = _prefill_args()
    d["out"] = _t([39, 8, 128], pa.PA_BF16)
    assert _prefill(lib, d) == -2                 # out like the query
    assert _prefill(lib, _prefill_args(T=0)) == 0  # no new tokens: nothing to do


def test_swap_blocks_rejects_bad_arguments(lib):
    r = ctypes.byref
    dev_k, dev_v = _t([32, 2, 16, 128], pa.PA_BF16), _t([32, 2, 16, 128], pa.PA_BF16)
    host_k, host_v = _t([64, 2, 16, 128], pa.PA_BF16), _t([64, 2, 16, 128], pa.PA_BF16)
    other = _t([64, 2, 8, 128], pa.PA_BF16)
    pairs = _t([3, 2], pa.PA_I64)
    assert lib.pa_swap_blocks(r(dev_k), r(dev_v), r(other), r(other), r(pairs), None) == -2
    assert lib.pa_swap_blocks(r(dev_k), r(dev_v), r(host_k), r(host_v), r(_t([3, 2], pa.PA_I32)), None) == -3
    assert lib.pa_swap_blocks(r(dev_k), r(dev_v), r(host_k), r(host_v), r(_t([3, 3], pa.PA_I64)), None) == -2
    assert lib.pa_swap_blocks(r(dev_k), r(dev_v), r(host_k), r(host_v), r(_t([0, 2], pa.PA_I64)), None) == 0


def test_fp8_entry_points_reject_bad_arguments(lib):
    r = ctypes.byref
    kc8, vc8 = _t([32, 2, 16, 128], pa.PA_FP8_E4M3), _t([32, 2, 16, 128], pa.PA_FP8_E4M3)
    key = _t([5, 2, 128], pa.PA_BF16)
    slots = _t([5], pa.PA_I64)
    ks, vs = _t([2], pa.PA_F32), _t([2], pa.PA_F32)
    w = lambda k=key, kc=kc8, s1=ks, s2=vs: lib.pa_reshape_and_cache_fp8(r(k), r(k), r(kc), r(kc), r(slots),
                                                                         r(s1), r(s2), None)
    assert w(s1=_t([2], pa.PA_F16)) == -3                         # scales must be fp32
    assert w(s1=_t([3], pa.PA_F32), s2=_t([3], pa.PA_F32)) == -2   # one scale per kv head
    assert w(kc=_t([32, 2, 16, 128], pa.PA_BF16)) == -3            # the caches must be FP8
    # the 16-bit entry points refuse FP8 caches, whose values need their scales
    a = _decode_args()
    a["kc"], a["vc"] = kc8, vc8
    assert _decode(lib, a) == -3
    S, Hq = 4, 8

    def dec(q_dt=pa.PA_BF16, s1=ks, flags=0, kc=kc8, D=128):
        o, q = _t([S, Hq, D], pa.PA_F32), _t([S, Hq, D], q_dt)
        bt, cl = _t([S, 4], pa.PA_I32), _t([S], pa.PA_I32)
        return lib.pa_decode_fp8(r(o), r(q), r(kc), r(kc), r(bt), r(cl), r(s1), r(vs), 0.1, 16, 2, 0,
                                 flags, None, 0, None)

    assert dec(q_dt=pa.PA_F32) == -3                   # the query must be bf16 or fp16
    assert dec(s1=_t([2], pa.PA_F16)) == -3            # scales must be fp32
    assert dec(flags=pa.PA_DECODE_CUDA_CORES) == -4    # FP8 is read by the tensor-core kernel only
    assert dec(kc=_t([32, 2, 16, 64], pa.PA_FP8_E4M3), D=64) == -4  # head_dim 64 is not built
    assert pa.pa_last_error()


def _shared_call(lib, a, gs, pl, bs=16, hkv=2):
    r = ctypes.byref
    return lib.pa_decode_shared_prefix(r(a["out"]), r(a["query"]), r(a["kc"]), r(a["vc"]),
                                       r(a["bt"]), r(a["cl"]), r(gs) if gs is not None else None,
                                       r(pl), 0.1, bs, hkv, None, 0, None)


def test_shared_prefix_rejects_bad_arguments_before_cuda(lib):
    a = _decode_args()  # 4 sequences
    gs, pl = _t([2], pa.PA_I32), _t([4], pa.PA_I32)
    assert _shared_call(lib, a, None, pl) == -1                           # no group_start
    assert _shared_call(lib, a, _t([2], pa.PA_I64), pl) == -3             # group_start not int32
    assert _shared_call(lib, a, gs, _t([3], pa.PA_I32)) == -2             # not one per sequence
    assert _shared_call(lib, a, _t([0], pa.PA_I32), pl) == -2             # no entries at all
    assert _shared_call(lib, a, gs, _t([4], pa.PA_I32, stride=[2])) == -7  # not contiguous
    assert _shared_call(lib, _decode_args(dt=pa.PA_F32), gs, pl) == -4    # fp32 caches
    assert _shared_call(lib, a, gs, pl, bs=8) == -2                       # block_size disagrees
    assert pa.pa_last_error()


def test_shared_prefix_workspace_bytes(lib):
    # the decode workspace at the largest default worker count, then (m, l) and O / l of every
    # (sequence, query head) and 512-position prefix item, each region rounded up to 256 bytes
    def up(x):
        return (x + 255) // 256 * 256

    S, Hq, Hkv, D, MB, bs = 8, 32, 8, 128, 40, 16
    base = pa.pa_decode_workspace_bytes(S, Hq, Hkv, D, 0)
    if base == 0:  # no device: the default worker count is unknown, nothing to check
        assert pa.pa_decode_shared_prefix_workspace_bytes(S, Hq, Hkv, D, MB, bs) == 0
        return
    splits = (MB * bs + 511) // 512
    expect = up(base) + up(S * Hq * splits * 2 * 4) + up(S * Hq * splits * D * 4)
    assert pa.pa_decode_shared_prefix_workspace_bytes(S, Hq, Hkv, D, MB, bs) == expect
