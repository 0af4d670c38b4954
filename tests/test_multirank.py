"""The N > 1 host path of bench.py on CPU: two gloo ranks (127.0.0.1). The decode path does not
shard across GPUs (every (sequence, head) tile is independent), so N GPUs run N replicas of the
workload with no data-path collective; the only collective is the max over ranks of the timed
region, and the job's throughput counts every rank's tiles."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [3.5, 7.25][rank]
        slowest = bench.max_over_ranks(mine, world, "cpu")
        again = bench.max_over_ranks(mine * 0.5, world, "cpu")      # a second collective, same order
        out[rank] = (slowest, again, bench.job_throughput(world, 2048, 100, slowest))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    import torch.multiprocessing as mp
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:   # no fork of a process that may run OpenMP threads
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    slowest, again, value = res[0]
    assert slowest == 7.25 and again == 3.625
    assert value == pytest.approx(2 * 2048 * 100 / 7.25e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0
    assert bench.job_throughput(1, 10, 5, 2.0) == pytest.approx(25000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun the oracle arm is printed by rank 0; the other ranks exit 0 at once."""
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    assert bench.main() == 0
    assert capsys.readouterr().out == ""


def test_gpus_two_outside_torchrun_starts_two_ranks():
    """``bench.py --gpus 2`` run directly (no torchrun environment) starts two ranks itself
    (torch.distributed.run, 127.0.0.1); rank 0 prints one line with n_gpus = 2 -- here through the
    oracle arm, which needs no GPU; the other rank exits without output."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR",
                                                            "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--workload", "0", "--steps", "2", "--warmup", "1"],
                         env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["n_gpus"] == 2 and rec["impl"] == "reference"
