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
    with mp.Manager() as m:
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
