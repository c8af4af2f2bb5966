"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The attention path has no exchange step, so several GPUs run independent
replicas; what is shared is the timing rule (the slowest rank sets the time,
an element-wise max over ranks) and the whole-job throughput.  These tests run
that logic with two gloo ranks, and the reference arm under torchrun, where
only rank 0 runs the oracle and prints."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        got = bench.max_over_ranks(dist, [rank + 1.0, 5.0 - rank, 0.25 * rank], "cpu")
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(got, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        with open(tmp_path / f"rank{r}.json") as f:
            assert json.load(f) == [2.0, 5.0, 0.25]


def test_max_over_ranks_without_group_is_identity():
    assert bench.max_over_ranks(None, [3, 1.5], "cpu") == [3.0, 1.5]


def test_job_throughput_counts_every_replica():
    # two replicas of a 1e12-FLOP step, slowest rank 500 ms -> 4 TFLOP/s for the job
    assert abs(bench.job_tflops(2, 1e12, 500.0) - 4.0) < 1e-12
    assert abs(bench.job_tflops(1, 1e12, 500.0) - 2.0) < 1e-12


def test_reference_arm_under_torchrun_prints_once(tmp_path):
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0", "--config", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=str(tmp_path), env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2 and line["steps"] == 1
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
