"""FP8 E4M3 KV cache on the GPU: the quantising write is bit-exact with the oracle on every
bf16 value (and samples of fp32 / fp16 sources); the decode over FP8 caches matches the oracle's
attention over the decoded codes times the per-head scales, within the tolerance of 16-bit
caches, for every built block size and group size and for the worker counts and flags of the
16-bit tests; block copies and swaps move FP8 blocks as bytes."""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import (assert_bf16_output, assert_close, assert_no_device_error,
                               value_spread,
                               require_gpu, to_host, to_torch)

pytestmark = pytest.mark.gpu
FP8 = torch.float8_e4m3fn


def _codes(t):
    return t.view(torch.uint8).cpu().numpy()


def _all_tokens(b):
    """Rows and slots of every token of every sequence (the whole context through the write)."""
    ks, vs, slots = [], [], []
    for s in range(b.num_seqs):
        L = int(b.context_lens[s])
        if L == 0:
            continue
        t = np.arange(L)
        slots.append(b.block_tables[s, t // b.block_size].astype(np.int64) * b.block_size
                     + t % b.block_size)
        ks.append(b.logical_key[s][:L])
        vs.append(b.logical_value[s][:L])
    return np.concatenate(ks), np.concatenate(vs), np.concatenate(slots)


def _scales(rows, hkv, squeeze=1.0):
    """One scale per kv head: the head's largest magnitude maps to about 240 (the last head's
    to about 240 * squeeze, so squeeze > 1 saturates part of it)."""
    x = np.abs(W.decode_to_f64(rows, "bf16")).reshape(-1, hkv, rows.shape[-1])
    m = x.max(axis=(0, 2))
    sc = (m / 240.0).astype(np.float32)
    sc[-1] = np.float32(sc[-1] / squeeze)
    return np.maximum(sc, np.float32(1e-8))


class Fp8Batch:
    """An FP8 cache filled through both write paths (GPU kernel and oracle), NaN codes in every
    unused slot."""

    def __init__(self, oracle, b, squeeze=1.0):
        self.b = b
        nb, hkv, bs, d = b.key_cache.shape
        k, v, slots = _all_tokens(b)
        self.ks = _scales(k, hkv, squeeze)
        self.vs = _scales(v, hkv, squeeze)
        self.okc = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
        self.ovc = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
        assert oracle.reshape_and_cache_fp8(k, v, "bf16", self.okc, self.ovc, slots, self.ks,
                                            self.vs) == 0
        self.kc = torch.full((nb, hkv, bs, d), 0x7f, dtype=torch.uint8, device="cuda").view(FP8)
        self.vc = torch.full((nb, hkv, bs, d), 0x7f, dtype=torch.uint8, device="cuda").view(FP8)
        self.k_scale = torch.from_numpy(self.ks).cuda()
        self.v_scale = torch.from_numpy(self.vs).cuda()
        pa.pa_reshape_and_cache_fp8(to_torch(k, "bf16"), to_torch(v, "bf16"), self.kc, self.vc,
                                    to_torch(slots), self.k_scale, self.v_scale)
        self.query = to_torch(b.query, "bf16")
        self.tables = to_torch(b.block_tables)
        self.lens = to_torch(b.context_lens)

    def oracle_out(self, oracle):
        b = self.b
        return oracle.decode(b.query, self.okc, self.ovc, b.block_tables, b.context_lens, b.scale,
                             "fp8", q_dtype="bf16", k_scale=self.ks, v_scale=self.vs)

    def decode(self, out_dtype="f32", num_workers=0, flags=0, workspace=None):
        b = self.b
        out = torch.full(self.query.shape, float("nan"),
                         dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16, device="cuda")
        pa.pa_decode_fp8(out, self.query, self.kc, self.vc, self.tables, self.lens, self.k_scale,
                         self.v_scale, b.scale, b.block_size, b.num_kv_heads, num_workers, flags,
                         workspace)
        return to_host(out, out_dtype)


def test_fp8_write_every_bf16_value(oracle):
    """All 65,536 bf16 bit patterns (NaN and infinities included) through the write kernel with
    four different head scales: the codes equal the oracle's."""
    require_gpu()
    hkv, d = 4, 128
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16).reshape(-1, hkv, d)  # [128, 4, 128]
    rng = np.random.default_rng(4)
    vbits = bits[rng.permutation(bits.shape[0])]
    T = bits.shape[0]
    nb, bs = T // 16, 16
    slots = np.arange(T, dtype=np.int64)
    ks = np.array([1.0, 0.0078125, 0.37, 3.0], np.float32)
    vs = np.array([0.5, 1.7, 1e-3, 96.0], np.float32)
    okc = np.zeros((nb, hkv, bs, d), np.uint8)
    ovc = np.zeros((nb, hkv, bs, d), np.uint8)
    oracle.reshape_and_cache_fp8(bits, vbits, "bf16", okc, ovc, slots, ks, vs)
    kc = torch.zeros((nb, hkv, bs, d), dtype=torch.uint8, device="cuda").view(FP8)
    vc = torch.zeros_like(kc)
    pa.pa_reshape_and_cache_fp8(to_torch(bits, "bf16"), to_torch(vbits, "bf16"), kc, vc,
                                to_torch(slots), torch.from_numpy(ks).cuda(),
                                torch.from_numpy(vs).cuda())
    got_k, got_v = _codes(kc), _codes(vc)
    bad = np.nonzero(got_k.reshape(-1) != okc.reshape(-1))[0]
    assert bad.size == 0, f"{bad.size} key codes differ, e.g. {got_k.reshape(-1)[bad[:4]]} vs {okc.reshape(-1)[bad[:4]]}"
    assert np.array_equal(got_v, ovc)
    assert_no_device_error()


@pytest.mark.parametrize("src", ["f32", "f16"])
def test_fp8_write_other_sources(oracle, src):
    require_gpu()
    hkv, d, T = 2, 128, 64
    rng = np.random.default_rng(9)
    x = (rng.standard_normal((T, hkv, d)) * np.exp(rng.uniform(-12, 9, (T, hkv, d)))).astype(np.float32)
    x = x.astype(np.float16) if src == "f16" else x
    slots = rng.permutation(T * 2)[:T].astype(np.int64)
    slots[3] = -1
    ks = np.array([0.05, 2.5], np.float32)
    okc = np.zeros((8, hkv, 16, d), np.uint8)
    ovc = np.zeros((8, hkv, 16, d), np.uint8)
    oracle.reshape_and_cache_fp8(x, x, src, okc, ovc, slots, ks, ks[::-1].copy())
    kc = torch.zeros((8, hkv, 16, d), dtype=torch.uint8, device="cuda").view(FP8)
    vc = torch.zeros_like(kc)
    pa.pa_reshape_and_cache_fp8(torch.from_numpy(x).cuda(), torch.from_numpy(x).cuda(), kc, vc,
                                torch.from_numpy(slots).cuda(), torch.from_numpy(ks).cuda(),
                                torch.from_numpy(ks[::-1].copy()).cuda())
    assert np.array_equal(_codes(kc), okc) and np.array_equal(_codes(vc), ovc)


@pytest.fixture(scope="module")
def llama_fp8(oracle):
    b = W.build_batch("fp8", W.llama3_8b_decode(num_seqs=12, min_len=1, max_len=300).context_lens,
                      num_heads=32, num_kv_heads=8, head_dim=128, block_size=16, dtype="bf16",
                      seed=W.BASE_SEED + 720, keep_logical=True)
    fb = Fp8Batch(oracle, b, squeeze=3.0)
    return fb, fb.oracle_out(oracle)


def test_fp8_caches_equal_the_oracles(llama_fp8):
    require_gpu()
    fb, _ = llama_fp8
    assert np.array_equal(_codes(fb.kc), fb.okc) and np.array_equal(_codes(fb.vc), fb.ovc)


@pytest.mark.parametrize("workers,flags", [(0, 0), (1, 0), (7, 0), (33, 0), (512, 0), (7, 1),
                                           (0, 1), (0, 4), (33, 5)])
def test_fp8_decode(llama_fp8, workers, flags):
    require_gpu()
    fb, ref = llama_fp8
    out = fb.decode("f32", workers, flags)
    assert_close(out, ref, "bf16", f"fp8 W={workers} flags={flags}")
    outb = fb.decode("bf16", workers, flags)
    spread = value_spread(fb.ovc, "fp8", fb.b.block_tables, fb.b.context_lens, ref,
                          fb.b.block_size, v_scale=fb.vs)
    assert_bf16_output(outb, ref, f"fp8 bf16 out W={workers} flags={flags}", spread)
    assert_no_device_error()


@pytest.mark.parametrize("bs,hq,hkv", [(8, 8, 8), (16, 16, 8), (32, 32, 4), (16, 64, 8), (8, 16, 2)])
def test_fp8_decode_configurations(oracle, bs, hq, hkv):
    require_gpu()
    lens = [1, 15, 16, 17, 100, 257, 600, 0, 33]
    b = W.build_batch("fp8cfg", lens, num_heads=hq, num_kv_heads=hkv, head_dim=128,
                      block_size=bs, dtype="bf16", seed=W.BASE_SEED + 730 + bs + hq,
                      keep_logical=True)
    fb = Fp8Batch(oracle, b)
    ref = fb.oracle_out(oracle)
    for workers in (0, 3):
        assert_close(fb.decode("f32", workers), ref, "bf16", f"fp8 bs{bs} G{hq // hkv} W={workers}")
    assert_no_device_error()


def test_fp8_blocks_copy_and_swap():
    require_gpu()
    src = torch.randint(0, 256, (20, 4, 16, 128), dtype=torch.uint8, device="cuda").view(FP8)
    srcv = torch.randint(0, 256, (20, 4, 16, 128), dtype=torch.uint8, device="cuda").view(FP8)
    host_k = torch.zeros((6, 4, 16, 128), dtype=torch.uint8).pin_memory().view(FP8)
    host_v = torch.zeros((6, 4, 16, 128), dtype=torch.uint8).pin_memory().view(FP8)
    pa.pa_swap_blocks(src, srcv, host_k, host_v, torch.tensor([[19, 0], [3, 5]], device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(host_k.view(torch.uint8)[0], src.view(torch.uint8)[19].cpu())
    assert torch.equal(host_v.view(torch.uint8)[5], srcv.view(torch.uint8)[3].cpu())
    pa.pa_copy_blocks(src, srcv, torch.tensor([[2, 7]], device="cuda"))
    assert torch.equal(src.view(torch.uint8)[7], src.view(torch.uint8)[2])
    assert_no_device_error()


def test_fp8_refusals():
    require_gpu()
    kc = torch.zeros((4, 2, 16, 128), dtype=torch.uint8, device="cuda").view(FP8)
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((2, 4, 128), dtype=torch.float32, device="cuda")
    tables = torch.zeros((2, 4), dtype=torch.int32, device="cuda")
    lens = torch.ones(2, dtype=torch.int32, device="cuda")
    sc = torch.ones(2, dtype=torch.float32, device="cuda")
    with pytest.raises(pa.PagedAttentionError) as info:  # FP8 caches without scales
        pa.pa_decode_ex(out, q, kc, kc, tables, lens, 0.1, 16, 2)
    assert info.value.status == pa.PA_ERR_DTYPE
    with pytest.raises(pa.PagedAttentionError) as info:  # CUDA-core kernel
        pa.pa_decode_fp8(out, q, kc, kc, tables, lens, sc, sc, 0.1, 16, 2, flags=pa.PA_DECODE_CUDA_CORES)
    assert info.value.status == pa.PA_ERR_UNSUPPORTED
    with pytest.raises(pa.PagedAttentionError) as info:  # one scale per kv head
        pa.pa_decode_fp8(out, q, kc, kc, tables, lens, sc[:1], sc, 0.1, 16, 2)
    assert info.value.status == pa.PA_ERR_SHAPE
    kc64 = torch.zeros((4, 2, 16, 64), dtype=torch.uint8, device="cuda").view(FP8)
    with pytest.raises(pa.PagedAttentionError) as info:  # head_dim 64 not built
        pa.pa_decode_fp8(out[..., :64].contiguous(), q[..., :64].contiguous(), kc64, kc64, tables,
                         lens, sc, sc, 0.1, 16, 2)
    assert info.value.status == pa.PA_ERR_UNSUPPORTED
