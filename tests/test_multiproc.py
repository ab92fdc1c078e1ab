"""The benchmark's multi-rank plumbing on CPU with gloo, world size 2: ranks meet at a
barrier, the job time is the max over ranks, and the whole-job rate counts every rank's
work over that time (weak scaling: each GPU runs the full workload on its own batch)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(dist)
        t = bench.max_over_ranks(dist, 10.0 + 5.0 * rank)  # rank 1 is slower
        rate = bench.job_throughput(100.0, world, t * 4, 4)
        q.put((rank, t, rate))
        bench.barrier(dist)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, rate in res:
        assert t == 15.0                       # the slowest rank's time, seen by both
        assert rate == pytest.approx(2 * 100.0 / (15.0 / 1e3))


def test_world_size_must_match_gpus(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.dist_setup(1)


def test_reference_arm_line(capsys, monkeypatch):
    """--impl reference times the oracle on host cores and prints the reference line."""
    import json
    import sys

    import bench
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--steps", "1",
                                      "--warmup", "3", "--B", "1", "--Sq", "128", "--Sk", "128",
                                      "--Hq", "4", "--Hk", "2"])
    monkeypatch.delenv("RANK", raising=False)
    bench.main()
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["unit"] == "TFLOP/s"
