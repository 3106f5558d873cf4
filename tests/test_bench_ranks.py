"""The multi-rank plumbing of bench.py, on CPU: two gloo ranks.

With N GPUs the benchmark runs N independent replicas (the block does not
shard); the only collectives are a barrier around the timed region and the
max over ranks of the measured time.  These tests run that logic as two
processes on 127.0.0.1 with the gloo backend, and check that the reference
arm does no work on a rank other than 0.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(world, 1.0 + 10.0 * rank, device="cpu")  # rank 1 is slower
        bench.barrier(world)
        out.put((rank, ms, bench.job_us_per_layer(ms, steps=5, layers=47, world=world)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=10) for _ in range(world))
    assert [r for r, _, _ in res] == [0, 1]
    assert all(ms == 11.0 for _, ms, _ in res)  # every rank reports the slowest
    # 2 replicas x 5 steps x 47 layers of work in 11 ms
    assert all(us == pytest.approx(11.0e3 / (5 * 47) / 2) for _, _, us in res)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(1, 3.5) == 3.5
    bench.barrier(1)
    assert bench.job_us_per_layer(2.0, steps=4, layers=47, world=1) == pytest.approx(2e3 / 188)


def test_reference_arm_does_nothing_on_other_ranks(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"batch": 4, "steps": 1, "warmup": 0, "gpus": 2, "layers": 47})()
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""
