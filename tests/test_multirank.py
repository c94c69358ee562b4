"""Multi-rank host logic of bench.py on CPU: two gloo ranks (127.0.0.1).

The benchmark runs one replica of the decode-step stream per GPU (the
problems are independent: no data-path collective); the only cross-rank
steps are barriers and the max of the ranks' times, and the reported value
is the bytes of all ranks over the slowest rank's time.
"""
import datetime
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], world, "cpu")
        gbs = bench.job_gbs(2_000_000, 10, world, ms)
        # a second reduction in the same order on every rank
        ms2 = bench.max_over_ranks(times[rank] / 2, world, "cpu")
        dist.barrier()
        out.put((rank, ms, gbs, ms2))
    finally:
        dist.destroy_process_group()


def _run(world, times):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_two_ranks_take_the_slowest_time():
    res = _run(2, [3.0, 5.0])
    assert [r[0] for r in res] == [0, 1]
    for _, ms, gbs, ms2 in res:
        assert ms == 5.0
        assert ms2 == 2.5
        # all ranks' bytes over the slowest rank's time (weak scaling)
        assert gbs == pytest.approx(2_000_000 * 10 * 2 / 5e-3 * 1e-9)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_gbs(1_000_000, 4, 1, 2.0) == pytest.approx(2.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    class A:
        tau, steps, warmup, gpus = 3.0, 1, 3, 2
    monkeypatch.setenv("RANK", "1")
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""
