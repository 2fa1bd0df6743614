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


def test_reference_arm_line_keeps_the_contract(monkeypatch, capsys):
    """Rank 0 of the reference arm (the oracle on the host) prints one JSON line with the contract's keys."""
    import json

    import bench

    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    for wl in ("tiny",):  # the small workload: a few seconds of oracle work
        assert bench.run_reference(bench.parse_args(["--impl", "reference", "--workload", wl, "--steps", "1",
                                                     "--warmup", "3"])) == 0
        lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
        assert len(lines) == 1
        d = json.loads(lines[0])
        for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                    "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
            assert key in d, key
        assert d["impl"] == "reference" and d["value"] > 0 and d["config"]["workload"] == wl
        assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
        assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_mxfp4_oracle_step_uses_decoded_weights():
    """The CPU baseline of an MXFP4 workload computes with the weights the encoding represents."""
    import numpy as np

    import bench
    import oracle
    import synth

    wl = synth.workload("tiny", weights="mxfp4")
    step = bench.OracleStep(wl)
    step.prepare(8)
    e = next(i for i, g in enumerate(step.gu) if g is not None)
    raw = synth.w_gateup_expert_host(wl, e)
    assert (step.gu[e] == oracle.mxfp4_round_trip(raw)).all()
    assert not (step.gu[e] == raw).all()
    out = step.run(8)
    assert out.shape == (8, wl.d) and np.isfinite(out).all()
