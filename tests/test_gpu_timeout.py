"""A wait on a copy that can never complete ends, records PA_DEVERR_TIMEOUT and leaves the
CUDA context usable.

The child process sets two test hooks of the library: PA_TEST_STALL_COPIES=1 makes each decode
warp's first stage expect 16 bytes that no copy delivers, and PA_TEST_WAIT_LIMIT_CYCLES
shortens every wait to about a millisecond.  Every copy that was issued still lands (the
warp waits for each before it returns); nothing faults or hangs.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import torch
import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import DeviceBatch
pa.pa_get_device_error(clear=True)
b = W.llama3_8b_decode(num_seqs=8, min_len=64, max_len=600)
db = DeviceBatch(b)
db.write()
db.decode("f32")
torch.cuda.synchronize()
flags = pa.pa_get_device_error(clear=True)
assert flags & pa.PA_DEVERR_TIMEOUT, hex(flags)
pa.pa_release_workspaces()           # the merge counters may hold partial counts: start afresh
x = torch.arange(1000, device="cuda", dtype=torch.float32)
assert float(x.sum().item()) == 499500.0
torch.cuda.synchronize()
print("timeout recorded, context usable")
"""


def test_stalled_copy_times_out_and_context_survives():
    env = dict(os.environ, PA_TEST_STALL_COPIES="1", PA_TEST_WAIT_LIMIT_CYCLES="2000000")
    res = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "context usable" in res.stdout
