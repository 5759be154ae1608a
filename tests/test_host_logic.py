"""Host-side logic of the parity checks and of bench.py, on CPU: the bf16-output bound of
tests/gpu_helpers.py on the oracle's own output, and the summaries bench.py computes from
per-launch times and decode timelines."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import paged_kv_cache_427_b200 as pa  # noqa: E402
from paged_kv_cache_427_b200 import workloads as W  # noqa: E402
from tests import gpu_helpers  # noqa: E402
from tests.gpu_helpers import assert_bf16_output, oracle_step, value_spread  # noqa: E402


@pytest.fixture(autouse=True)
def _keep_gpu_figures_only():
    """The checks below run on synthetic outputs: keep them out of the GPU parity summary."""
    n = len(gpu_helpers.RESULTS)
    yield
    del gpu_helpers.RESULTS[n:]


@pytest.fixture(scope="module")
def small(oracle):
    b = W.llama3_8b_decode(num_seqs=6, min_len=1, max_len=200)
    ref, kc, vc = oracle_step(oracle, b)
    return b, ref, vc


def test_spread_is_the_largest_distance_of_a_context_value(small):
    b, ref, vc = small
    sp = value_spread(vc, b.dtype, b.block_tables, b.context_lens, ref, b.block_size)
    s, h, d = 2, 5, 17
    L = int(b.context_lens[s])
    g = h // (b.num_heads // b.num_kv_heads)
    v = [W.decode_to_f64(vc[b.block_tables[s, t // b.block_size], g, t % b.block_size, d], "bf16")
         for t in range(L)]
    assert sp[s, h, d] == max(abs(x - ref[s, h, d]) for x in v)


def test_bf16_bound_accepts_the_rounded_oracle_and_rejects_two_ulps(small):
    b, ref, vc = small
    sp = value_spread(vc, b.dtype, b.block_tables, b.context_lens, ref, b.block_size)
    rne = W.f32_to_bf16_bits(ref.astype(np.float32))
    assert assert_bf16_output(rne, ref, "rounded oracle", sp) == 1.0
    bad = rne.copy()
    bad.flat[7] += 2  # two ulps away
    with pytest.raises(AssertionError):
        assert_bf16_output(bad, ref, "two ulps off", sp)
    # 2% of the elements set to the other bf16 neighbour of the exact value: each within one
    # ulp (inside the bound), but too many differ from the nearest-even rounding
    trunc = (ref.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)  # toward zero
    other = np.where(rne == trunc, trunc + np.uint16(1), trunc).astype(np.uint16)
    off = rne.copy()
    off.flat[: off.size // 50] = other.flat[: off.size // 50]
    with pytest.raises(AssertionError, match="equal RNE"):
        assert_bf16_output(off, ref, "2% one ulp off", sp)


def test_launch_stats():
    st = bench.launch_stats([0.05, 0.06, 0.04, 0.05])
    assert st == {"mean_launch_us": 50.0, "median_launch_us": 50.0, "min_launch_us": 40.0,
                  "launches": 4}


def test_timeline_summary_of_synthetic_launches():
    """Two launches of 6 warps on 3 SMs: start 0.1 w us, first tile at 5 us, last tile at
    40 + w us, done 1 us later, the merge warp 0.5 us after that; the SMs finish in the same
    order both times."""
    recs = []
    base = 1_700_000_000_000_000_000
    for launch in range(2):
        r = np.zeros((6, pa.TIMELINE_WORDS), np.int64)
        for w in range(6):
            r[w, pa.TL_START] = base + 100 * w
            r[w, pa.TL_ISSUE] = base + 3000
            r[w, pa.TL_FIRST] = base + 5000
            r[w, pa.TL_LAST] = base + 40000 + 1000 * w
            r[w, pa.TL_DONE] = base + 41000 + 1000 * w
            r[w, pa.TL_MERGED] = base + 41500 + 1000 * w
            r[w, pa.TL_SM] = w // 2
            r[w, pa.TL_CHUNKS] = 10
        recs.append(r.reshape(-1))
    s = bench.timeline_summary(recs, chunk_bytes=8192)
    assert s["launches"] == 2
    assert s["first_tile_us_p50"] == 5.0
    assert s["end_us"] == 46.5
    assert s["issue_us_p50"] == 3.0
    assert s["tail_us"] == pytest.approx(46.5 - 44.0)
    assert s["sm_finish_rank_corr"] == 1.0
    assert s["sm_finish_us_min_p50_max"] == [42.5, 44.5, 46.5]
    rates = sum(10 * 8192 / ((35 + w) * 1e-6) / 1e9 for w in range(6))
    assert s["sum_of_warp_rates_GBps"] == pytest.approx(rates, abs=0.01)


def test_default_run_measures_every_config():
    names = [n for n, _ in bench.CONFIG_RUNS]
    for n in ("long_mixed", "short_chat_bs8", "short_chat_bs16", "short_chat_bs32", "shared_prefix",
              "chunked_prefill"):
        assert n in names
    assert ("llama3_8b_decode", "fp8") in bench.CONFIG_RUNS
    assert ("shared_prefix", "shared") in bench.CONFIG_RUNS
