"""pa_decode_step_fp8: the quantising cache write and the decode over FP8 caches in one call (one
kernel when each sequence brings one token in the query's type).  Against the oracle: the caches
after the step are bit-exact with the oracle's quantising write of the same tokens (so the fused
kernel stores the same codes as pa_reshape_and_cache_fp8), and the output matches the oracle's
decode over those caches within the tolerance of 16-bit caches."""
import numpy as np
import pytest
import torch

import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import assert_close, assert_no_device_error, require_gpu, to_host, to_torch
from tests.test_gpu_fp8 import FP8, _codes, _scales

pytestmark = pytest.mark.gpu


def _slot(b, s, t):
    return int(b.block_tables[s, t // b.block_size]) * b.block_size + t % b.block_size


class StepCase:
    """FP8 caches holding positions 0 .. L-2 of every sequence (written through both paths); the
    step brings position L-1 of each."""

    def __init__(self, oracle, lens, bs=16, hq=32, hkv=8, seed=0, key_dtype="bf16"):
        b = W.build_batch("fp8step", np.asarray(lens, np.int32), num_heads=hq, num_kv_heads=hkv,
                          head_dim=128, block_size=bs, dtype="bf16",
                          seed=W.BASE_SEED + 1100 + seed, keep_logical=True)
        self.b = b
        nb, _, _, d = b.key_cache.shape
        rows_k, rows_v, slots = [], [], []
        for s in range(b.num_seqs):
            L = int(b.context_lens[s])
            for t in range(max(L - 1, 0)):
                slots.append(_slot(b, s, t))
            rows_k.append(b.logical_key[s][:max(L - 1, 0)])
            rows_v.append(b.logical_value[s][:max(L - 1, 0)])
        k_old, v_old = np.concatenate(rows_k), np.concatenate(rows_v)
        slots = np.asarray(slots, np.int64)
        all_k = np.concatenate([b.logical_key[s][:int(b.context_lens[s])] for s in range(b.num_seqs)])
        self.ks, self.vs = _scales(all_k, hkv, 2.0), _scales(all_k, hkv, 1.0)
        self.okc = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
        self.ovc = np.full((nb, hkv, bs, d), 0x7f, np.uint8)
        if len(slots):
            assert oracle.reshape_and_cache_fp8(k_old, v_old, "bf16", self.okc, self.ovc, slots,
                                                self.ks, self.vs) == 0
        self.kc = torch.full((nb, hkv, bs, d), 0x7f, dtype=torch.uint8, device="cuda").view(FP8)
        self.vc = torch.full((nb, hkv, bs, d), 0x7f, dtype=torch.uint8, device="cuda").view(FP8)
        self.k_scale = torch.from_numpy(self.ks).cuda()
        self.v_scale = torch.from_numpy(self.vs).cuda()
        if len(slots):
            pa.pa_reshape_and_cache_fp8(to_torch(k_old, "bf16"), to_torch(v_old, "bf16"), self.kc,
                                        self.vc, to_torch(slots), self.k_scale, self.v_scale)
        # the step's tokens: position L-1 of each sequence
        self.new_k = np.stack([b.logical_key[s][max(int(b.context_lens[s]) - 1, 0)]
                               for s in range(b.num_seqs)])
        self.new_v = np.stack([b.logical_value[s][max(int(b.context_lens[s]) - 1, 0)]
                               for s in range(b.num_seqs)])
        self.new_slots = np.array([_slot(b, s, int(b.context_lens[s]) - 1) if b.context_lens[s] > 0
                                   else -1 for s in range(b.num_seqs)], np.int64)
        self.key_dtype = key_dtype

    def run(self, oracle, workspace=None):
        b = self.b
        kd = self.key_dtype
        key = to_torch(self.new_k, "bf16") if kd == "bf16" else \
            torch.from_numpy(W.decode_to_f64(self.new_k, "bf16").astype(np.float32)).cuda()
        value = to_torch(self.new_v, "bf16") if kd == "bf16" else \
            torch.from_numpy(W.decode_to_f64(self.new_v, "bf16").astype(np.float32)).cuda()
        out = torch.full((b.num_seqs, b.num_heads, b.head_dim), float("nan"), dtype=torch.float32,
                         device="cuda")
        pa.pa_decode_step_fp8(key, value, self.kc, self.vc, to_torch(self.new_slots),
                              self.k_scale, self.v_scale, out, to_torch(b.query, "bf16"),
                              to_torch(b.block_tables), to_torch(b.context_lens), b.scale,
                              b.block_size, b.num_kv_heads, workspace=workspace)
        torch.cuda.synchronize()
        src = self.new_k if kd == "bf16" else W.decode_to_f64(self.new_k, "bf16").astype(np.float32)
        vsrc = self.new_v if kd == "bf16" else W.decode_to_f64(self.new_v, "bf16").astype(np.float32)
        assert oracle.reshape_and_cache_fp8(src, vsrc, kd, self.okc, self.ovc, self.new_slots,
                                            self.ks, self.vs) == 0
        ref = oracle.decode(b.query, self.okc, self.ovc, b.block_tables, b.context_lens, b.scale,
                            "fp8", q_dtype="bf16", k_scale=self.ks, v_scale=self.vs)
        return to_host(out, "f32"), ref


@pytest.mark.parametrize("bs,hq,hkv", [(16, 32, 8), (8, 16, 2), (32, 32, 4), (16, 64, 8)])
def test_fused_fp8_step_matches_the_oracle(oracle, bs, hq, hkv):
    require_gpu()
    lens = [1, 2, 15, 16, 17, 33, 100, 257, 600, 1200]
    case = StepCase(oracle, lens, bs, hq, hkv, seed=bs + hq)
    got, ref = case.run(oracle)
    assert np.array_equal(_codes(case.kc), case.okc), "key codes differ from the oracle's write"
    assert np.array_equal(_codes(case.vc), case.ovc), "value codes differ from the oracle's write"
    assert_close(got, ref, "bf16", f"fused fp8 step bs{bs} G{hq // hkv}")
    assert_no_device_error()


def test_fp8_step_full_size_with_caller_workspace(oracle):
    require_gpu()
    b = W.llama3_8b_decode()
    case = StepCase(oracle, b.context_lens, seed=7)
    n = pa.pa_decode_workspace_bytes(case.b.num_seqs, 32, 8, 128, 0)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    got, ref = case.run(oracle, workspace=ws)
    assert np.array_equal(_codes(case.kc), case.okc) and np.array_equal(_codes(case.vc), case.ovc)
    assert_close(got, ref, "bf16", "fused fp8 step, Llama-shaped batch (every sequence)")
    assert_no_device_error()


def test_fp8_step_with_fp32_tokens_takes_two_kernels(oracle):
    """key/value in fp32 (not the query's type): the write kernel, then the decode."""
    require_gpu()
    case = StepCase(oracle, [5, 40, 300, 1], key_dtype="f32", seed=3)
    got, ref = case.run(oracle)
    assert np.array_equal(_codes(case.kc), case.okc) and np.array_equal(_codes(case.vc), case.ovc)
    assert_close(got, ref, "bf16", "fp8 step, fp32 tokens")
    assert_no_device_error()


def test_fused_fp8_step_flags_a_slot_that_is_not_the_last_position(oracle):
    require_gpu()
    case = StepCase(oracle, [50, 60, 70, 80], seed=11)
    used = set()
    b = case.b
    for s in range(b.num_seqs):
        used.update(int(x) for x in b.block_tables[s, :(int(b.context_lens[s]) + 15) // 16])
    free = next(i for i in range(b.num_blocks) if i not in used)
    case.new_slots[2] = free * b.block_size
    pa.pa_get_device_error(clear=True)
    got, _ = case.run(oracle)
    assert pa.pa_get_device_error(clear=True) & pa.PA_DEVERR_SLOT
    # stored as asked (the oracle wrote the same slots)
    assert np.array_equal(_codes(case.kc), case.okc) and np.array_equal(_codes(case.vc), case.ovc)
    # every sequence attends to its token as position L-1 (the kernel reads it from the step's
    # rows, not from the slot): compare with the oracle's decode of caches that also hold
    # token 2 at sequence 2's position L-1
    okc, ovc = case.okc.copy(), case.ovc.copy()
    s2 = _slot(b, 2, int(b.context_lens[2]) - 1)
    assert oracle.reshape_and_cache_fp8(case.new_k[2:3], case.new_v[2:3], "bf16", okc, ovc,
                                        np.array([s2], np.int64), case.ks, case.vs) == 0
    ref = oracle.decode(b.query, okc, ovc, b.block_tables, b.context_lens, b.scale, "fp8",
                        q_dtype="bf16", k_scale=case.ks, v_scale=case.vs)
    assert_close(got, ref, "bf16", "fused fp8 step with one misplaced slot")
