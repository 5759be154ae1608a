"""The multi-rank side of bench.py on CPU: two gloo ranks take the element-wise maximum of
their times (the slowest rank's), and under torchrun the reference arm runs on rank 0 alone
while the other ranks exit 0 without output."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        q.put((rank, bench.max_over_ranks([1.0 + rank, 5.0 - rank, 3.0])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: [2.0, 5.0, 3.0], 1: [2.0, 5.0, 3.0]}


def test_max_over_ranks_without_a_group_returns_the_values():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1, 2.5]) == [1.0, 2.5]


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_prints_once():
    """Two ranks on CPU: rank 0 times the oracle and prints one JSON line, rank 1 does nothing."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny_fp32"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=560)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0


@pytest.mark.timeout(600)
def test_reference_arm_of_a_prefill_workload_times_the_prefill_oracle():
    """The reference arm reports the arm's own metric: TFLOP/s of the oracle's prefill for the
    chunked-prefill workload."""
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "chunked_prefill",
           "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=560)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads([l for l in res.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s"
    assert line["metric"].startswith("paged prefill attention") and line["value"] > 0


@pytest.mark.timeout(600)
@pytest.mark.parametrize("extra,unit", [(["--kv", "fp8"], "GB/s"), (["--swap"], "GB/s")])
def test_reference_arm_of_fp8_and_swap_runs_the_matching_oracle(extra, unit):
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"] + extra
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=560)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads([l for l in res.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["unit"] == unit and line["value"] > 0
    if "--swap" in extra:
        assert line["metric"].startswith("block swap")
    else:
        assert line["config"]["kv_dtype"] == "fp8_e4m3"
