"""Host logic of bench.py on CPU: the max-over-ranks timing and the whole-job throughput of N
replicas, run as two gloo ranks; the reference arm does no work on ranks other than 0."""
import io
import os
import socket
import contextlib

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [1200.0, 1500.0][rank]          # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms)
        out.put((rank, total, bench.job_throughput(2001, 5, world, total)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [1500.0, 1500.0]
    # 2 replicas x 2001 tokens x 5 steps in 1.5 s
    assert res[0][2] == pytest.approx(2 * 2001 * 5 / 1.5)


def test_single_process_keeps_its_own_time():
    assert bench.max_over_ranks(123.0) == 123.0
    assert bench.job_throughput(2001, 5, 1, 1000.0) == pytest.approx(10005.0)


def test_reference_arm_is_silent_on_other_ranks(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    a = type("A", (), {"workload": "c1", "steps": 1, "warmup": 0, "cpu_decode_steps": 1})()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(a)
    assert buf.getvalue() == ""
