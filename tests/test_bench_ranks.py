"""The multi-rank path of bench.py on CPU: two gloo ranks (replicas) agree on
the slowest rank's time and the whole-job throughput; the reference arm runs
on rank 0 only."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 * (rank + 1)          # rank 1 is the slow replica
        m = bench.max_over_ranks(ms, world, torch.device("cpu"))
        out[rank] = (m, bench.job_tokens_per_s(world, 4096, 20, m))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1]
    m, tps = out[0]
    assert m == 20.0
    assert tps == pytest.approx(2 * 4096 * 20 / 0.020)


def test_single_rank_needs_no_collective():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_tokens_per_s(1, 64, 10, 1000.0) == pytest.approx(640.0)


def test_reference_arm_only_on_rank_zero(monkeypatch, capsys):
    class A:
        workload, steps, warmup = "tiny_f32", 1, 0
    bench.run_reference(A, rank=1, world=2)   # other ranks exit without work
    assert capsys.readouterr().out == ""


def test_reference_arm_line_on_cpu(capsys):
    """--impl reference on the tiny workload: one JSON line from the oracle."""
    import json

    class A:
        workload, steps, warmup = "tiny_f32", 2, 1
    bench.run_reference(A, rank=0, world=1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["unit"] == "tokens/s"
