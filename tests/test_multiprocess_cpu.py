"""bench.py's multi-rank bookkeeping on CPU with gloo (world size 2): the step
time is the max over ranks and the value is the whole-job throughput."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 * (rank + 1)          # rank 1 is the slowest
        t = bench.reduce_step_time(ms, dist)
        v = bench.whole_job_value(1000, world, t)
        dist.barrier()
        q.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, v in res:
        assert t == pytest.approx(20.0)               # max over ranks
        assert v == pytest.approx(2 * 1000 / 0.020)   # all ranks' units / slowest time


def test_single_rank_identity():
    import bench
    assert bench.reduce_step_time(3.5, None) == 3.5
    assert bench.whole_job_value(7, 1, 1.0) == pytest.approx(7000.0)


def test_reference_arm_non_zero_rank_exits_without_work(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), dict(warmup=3, steps=1, gpus=2, ref_frames=1))()
    assert bench.run_reference(args, bench.synth.CONFIGS["tiny_fp32"]) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_contract_line(monkeypatch, capsys):
    import json
    import bench
    monkeypatch.setenv("RANK", "0")
    args = type("A", (), dict(warmup=3, steps=2, gpus=1, ref_frames=2))()
    assert bench.run_reference(args, bench.synth.CONFIGS["tiny_fp32"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
