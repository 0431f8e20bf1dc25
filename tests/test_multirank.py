"""The N > 1 host path of bench.py on CPU with two gloo ranks: the decode
path does not shard (replicas only), so the only cross-rank steps are the
reduction of the timings (max over ranks) and of the work (sum over ranks),
and the reference arm, which rank 0 alone runs and prints."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _reduce_rank(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times, work = bench.reduce_over_ranks([1.0 + rank, 5.0 - rank, 0.25 * (rank + 1)],
                                              [10.0 * (rank + 1), 7.0], world, "cpu")
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"times": times, "work": work}, f)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_two_gloo_ranks(tmp_path):
    mp.spawn(_reduce_rank, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    for rank in range(2):
        with open(tmp_path / f"r{rank}.json") as f:
            r = json.load(f)
        assert r["times"] == [2.0, 5.0, 0.5]  # the slowest rank per figure
        assert r["work"] == [30.0, 14.0]      # every rank's work counted once


def test_reduce_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    times, work = bench.reduce_over_ranks([1.5, 2.5], [3.0], 1, "cpu")
    assert times == [1.5, 2.5] and work == [3.0]


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "3",
           "--cpu-budget", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
