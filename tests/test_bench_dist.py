"""Multi-process host logic of bench.py on CPU (gloo, world size 2): replicas report the max over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    r, local, w = bench.dist_init("gloo")
    assert (r, local, w) == (rank, rank, world)
    bench.barrier()
    out[rank] = bench.max_over_ranks(10.0 + 5.0 * rank)
    bench.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_process_is_identity():
    import bench

    assert bench.max_over_ranks(3.5) == 3.5
    bench.barrier()  # no process group: no-op


def test_reference_arm_on_other_ranks_does_no_work(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(bench.parse_args(["--impl", "reference", "--workload", "tiny"])) == 0
    assert capsys.readouterr().out == ""
