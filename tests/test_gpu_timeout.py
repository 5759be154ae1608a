"""A wait on a copy that can never complete ends, records PA_DEVERR_TIMEOUT and leaves the
CUDA context usable; reading the error word is then the whole recovery, for caller workspaces
and for the static scratch of pa_decode_noalloc alike.

The child process sets two test hooks of the library: PA_TEST_STALL_COPIES=1 makes each decode
warp's first stage expect 16 bytes that no copy delivers, and PA_TEST_WAIT_LIMIT_CYCLES
shortens every wait to about a millisecond.  With PA_TEST_STALL_COPIES=2 only the odd-numbered
worker warps stall, so the others finish their pieces and leave merge counters partly counted;
PA_TEST_STALL_CALLS limits the stall to the first decode launches of the process.  Every copy that was issued still lands (the
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


RECOVERY_CHILD = r"""
import sys
sys.path.insert(0, {root!r})
import torch
import paged_kv_cache_427_b200 as pa
from paged_kv_cache_427_b200 import workloads as W
from tests.gpu_helpers import DeviceBatch, assert_close, to_host
pa.pa_get_device_error(clear=True)
b = W.llama3_8b_decode(num_seqs=16, min_len=512, max_len=2048)
db = DeviceBatch(b)
db.write()
S, Hkv = b.num_seqs, b.num_kv_heads
n = pa.pa_decode_workspace_bytes(S, b.num_heads, Hkv, b.head_dim, 0)
ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
out = torch.empty(db.query.shape, dtype=torch.float32, device="cuda")

def ex():
    pa.pa_decode_ex(out, db.query, db.key_cache, db.value_cache, db.block_tables,
                    db.context_lens, b.scale, b.block_size, Hkv, workspace=ws)

def noalloc():
    pa.pa_decode_noalloc(out, db.query, db.key_cache, db.value_cache, db.block_tables,
                         db.context_lens, b.scale, b.block_size, Hkv)

# stalled launch 1 (caller workspace): the odd workers give up, the even ones take tickets
ex()
torch.cuda.synchronize()
counters = ws[: S * Hkv * 4].view(torch.int32)
left = int((counters != 0).sum())
assert left > 0, "the stalled call left no partly counted merge counter"
# stalled launch 2 (the static scratch of pa_decode_noalloc)
noalloc()
flags = pa.pa_get_device_error(clear=True)   # the recovery: read the error word
assert flags & pa.PA_DEVERR_TIMEOUT, hex(flags)
ref = to_host(db.decode("f32"), "f32")       # pa_decode, library-owned workspace
for name, call in (("pa_decode_ex", ex), ("pa_decode_noalloc", noalloc),
                   ("pa_decode_noalloc again", noalloc)):
    out.fill_(float("nan"))
    call()
    assert_close(to_host(out, "f32"), ref, "bf16", name + " after recovery")
assert int((counters != 0).sum()) == 0, "merge counters not left zero"
assert pa.pa_get_device_error(clear=True) == 0
print(f"recovered ({{left}} counters were left partly counted)")
"""


def test_timeout_recovery_of_workspaces_and_noalloc_scratch():
    env = dict(os.environ, PA_TEST_STALL_COPIES="2", PA_TEST_STALL_CALLS="2",
               PA_TEST_WAIT_LIMIT_CYCLES="2000000")
    res = subprocess.run([sys.executable, "-c", RECOVERY_CHILD.format(root=ROOT)], env=env,
                         capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "recovered" in res.stdout
