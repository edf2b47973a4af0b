"""Host logic of the benchmark's multi-GPU path, on CPU with the gloo backend.

bench.py runs one process per GPU; every rank is an independent replica on its
own seeded batch, and the only collectives are the timing barrier and the max
over ranks of the elapsed time.  These tests run that logic with world size 2
on CPU: the max over ranks, the whole-job throughput, disjoint per-rank
seeds, and the reference arm, which only rank 0 runs.
"""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        # each rank's "elapsed time" differs; every rank must see the largest
        elapsed = 10.0 + 5.0 * rank
        got = bench.max_over_ranks(elapsed, world)
        value = bench.job_throughput(world, 2.0e12, 10, got)
        with open(os.path.join(outdir, "rank%d.json" % rank), "w") as f:
            json.dump({"max": got, "value": value, "seeds": bench.rank_seeds(rank, 4)}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_world_size_2(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    assert all(r["max"] == 15.0 for r in res)                 # the slowest rank's time
    # whole-job TFLOP/s: both ranks' work over the slowest time, identical on every rank
    assert res[0]["value"] == res[1]["value"] == pytest.approx(2 * 2.0e12 * 10 / 15e-3 / 1e12)
    assert not set(res[0]["seeds"]) & set(res[1]["seeds"])    # each rank draws its own batch


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1, 1e12, 4, 2.0) == pytest.approx(2000.0)
    assert bench.job_throughput(8, 1e12, 4, 2.0) == pytest.approx(8 * 2000.0)   # weak scaling: work grows with N


def test_rank_seeds_are_disjoint_across_ranks_and_roles():
    seen = set()
    for rank in range(8):
        for base in (0, 100):
            s = bench.rank_seeds(rank, 4, base=base)
            assert not seen & set(s)
            seen |= set(s)


def test_reference_arm_runs_on_rank_0_only(monkeypatch, capsys):
    # under torchrun every rank starts the reference arm; ranks other than 0
    # return at once, without work and without printing
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"])
    called = []
    monkeypatch.setattr(bench, "run_reference", lambda args: called.append(args) or {})
    bench.main()
    assert called == [] and capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    bench.main()
    assert len(called) == 1
    assert json.loads(capsys.readouterr().out.strip()) == {}
