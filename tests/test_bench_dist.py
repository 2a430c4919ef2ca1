"""bench.py's multi-process plumbing on CPU: two gloo ranks (world size 2).

Each rank is an independent replica; the reported step time is the maximum
over ranks and the job's rate is the sum of the ranks' work over it.  The
reference arm runs on rank 0 only; other ranks exit without work.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 1.5 + rank  # rank 1 is the slow one
        got = bench.max_over_ranks(ms, world, dist, "cpu")
        results[rank] = (got, bench.whole_job_tflops(3e12, world, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(results)
    assert res[0][0] == res[1][0] == 2.5
    # 2 replicas x 3 TFLOP each in 2.5 ms
    assert res[0][1] == pytest.approx(2 * 3e12 / 2.5e-3 / 1e12)



def test_single_rank_is_identity():
    assert bench.max_over_ranks(4.25, 1) == 4.25
    assert bench.whole_job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)  # 1 TFLOP in 1 ms


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    called = []
    monkeypatch.setattr(bench.W, "inputs", lambda *a, **k: called.append(1))
    assert bench.run_reference(bench.parse_args(["--impl", "reference", "--gpus", "2"])) == 0
    assert not called


def test_reference_arm_line_on_rank0(monkeypatch, capsys):
    import json

    monkeypatch.setenv("RANK", "0")
    args = bench.parse_args(["--impl", "reference", "--workload", "C1", "--tokens", "8", "--steps", "2",
                             "--warmup", "1", "--cpu-threads", "2"])
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["steps"] == 2 and line["warmup"] == 1 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 2
    assert line["cpu_baseline"]["value"] == line["value"] == line["e2e"]["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert "C1" in line["config"]["workload"]
