"""The oracle still reproduces its stored record for the tiny fp32 workload bit for bit."""
import os

import numpy as np

from paged_kv_cache_427_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "tiny_fp32_oracle.txt")


def test_tiny_fp32_golden(oracle):
    b = workloads.tiny_fp32()
    kc, vc = b.key_cache.copy(), b.value_cache.copy()
    assert oracle.reshape_and_cache(b.key, b.value, kc, vc, b.slot_mapping, b.dtype) == 0
    out = oracle.decode(b.query, kc, vc, b.block_tables, b.context_lens, b.scale, b.dtype)
    ref = np.loadtxt(GOLDEN, dtype=np.float64).reshape(out.shape)
    np.testing.assert_array_equal(out, ref)
