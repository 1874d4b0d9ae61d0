"""The multi-GPU host logic of bench.py on the CPU: two gloo ranks.

The HSA path has no exchange step, so several GPUs run independent replicas; what
crosses ranks is only the barrier around the timed region and the max over ranks
of the measured times.  These tests run that logic with world size 2 on gloo, and
check that the reference arm does its work on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        barrier, allmax = bench.collectives(dist, "cpu")
        barrier()
        local_ms = 10.0 + 5.0 * rank               # each rank's own timing
        got = allmax(local_ms)
        barrier()
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as fh:
            fh.write(repr(got))
    finally:
        dist.destroy_process_group()


def test_two_rank_barrier_and_max_over_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    for r in range(2):
        assert float((tmp_path / f"rank{r}.txt").read_text()) == 15.0


def test_single_process_collectives_pass_through():
    sys.path.insert(0, ROOT)
    import bench
    barrier, allmax = bench.collectives(None, "cpu")
    barrier()
    assert allmax(3.5) == 3.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    called = []
    monkeypatch.setattr(bench, "run_reference", lambda args: called.append(args) or {})
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main() == 0
    assert called == []
    monkeypatch.setenv("RANK", "0")
    assert bench.main() == 0
    assert len(called) == 1
