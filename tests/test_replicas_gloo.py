"""The N > 1 path of bench.py, on CPU with gloo, world size 2.

The operator has no exchange between streams, so N GPUs run N independent
replicas (no collective on the data path).  What N > 1 adds is host
plumbing: ranks from the launcher's environment, a barrier around the timed
region, the MAX over ranks of the per-rank times, the whole-job rate over
all replicas, and distinct inputs per replica.  These tests run that
plumbing under ``torch.distributed.run`` as the driver launches bench.py,
on 127.0.0.1, with the gloo backend in place of NCCL.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_replicas_reduce_times_with_max_and_count_all_units(tmp_path):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}",
           os.path.join(ROOT, "tests", "gloo_replica_rank.py"), str(tmp_path)]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    recs = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    for i, rec in enumerate(recs):
        assert (rec["rank"], rec["world"], rec["local"]) == (i, 2, i)
        # rank 0 gave [10, 4, 7], rank 1 [11, 8, 6]: element-wise max on every rank
        assert rec["reduced"] == [11.0, 8.0, 7.0]
        # 2 replicas x 1000 units over the slowest replica's 11 ms
        assert rec["rate"] == pytest.approx(2 * 1000 / 11e-3)
        assert rec["inputs_reproducible"]
    assert recs[0]["inputs_equal_rank0"]
    assert not recs[1]["inputs_equal_rank0"]


def test_reference_arm_runs_on_rank_zero_only():
    """Under a multi-rank launch the oracle arm runs on rank 0 alone; the
    other ranks exit 0 without work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 1.5], 1, "cpu") == [3.0, 1.5]
    assert bench.job_rate(1, 500, 250.0) == pytest.approx(2000.0)
