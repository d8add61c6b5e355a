"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): the path shards into independent
replicas, so the only exchange is the max-over-ranks of the timings."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + 5.0 * rank, 2.0 - rank]  # rank 1 is slower on the first timing
        got = bench.max_over_ranks(local, "cpu")
        out[rank] = got + [bench.aggregate_steps_per_s(got[0], world)]
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_two_ranks():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1]
    assert out[0][:2] == [15.0, 2.0]
    assert out[0][2] == pytest.approx(2 * 1e3 / 15.0)


def test_single_process_is_identity():
    assert bench.max_over_ranks([3.0, 4.5], "cpu") == [3.0, 4.5]
    assert bench.aggregate_steps_per_s(2.0, 1) == 500.0


def test_reference_arm_only_runs_on_rank_zero(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr("sys.argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    bench.main()
    assert capsys.readouterr().out == ""
