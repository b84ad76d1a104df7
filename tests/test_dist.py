"""Multi-rank host logic of bench.py, on CPU with the gloo backend (world size 2).

bench.py runs one replica of the wave round per GPU (weak scaling); the only
cross-rank steps are a barrier and the max of the elapsed time, from which
rank 0 reports whole-job throughput. Those steps are exercised here without a
GPU.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        assert (ws, r, local) == (world, rank, rank)
        bench.barrier()
        elapsed = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.reduce_max(elapsed)
        out[rank] = got
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_reduce_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_reduce_max_without_process_group_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun the oracle arm prints from rank 0 alone; other ranks exit
    without work (and without a process group of their own)."""
    import argparse

    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.run_reference(argparse.Namespace(steps=1, warmup=3)) is None
    assert capsys.readouterr().out == ""
