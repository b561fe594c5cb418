"""Multi-rank host logic of the benchmark on CPU with gloo, world size 2:
each rank gets its own batch (weak scaling), the reported time is the slowest
rank's, and a rank that fails before the reduction makes the other rank fail
within the process group's timeout instead of waiting for ever."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from fp4_kv_cache_step_b200 import workloads as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s=20):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _worker_reduce(rank, world, port, q):
    _init(rank, world, port)
    try:
        w = bench.rank_workload(wl.DECODE_128K, rank)
        got = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        seeds = [None] * world
        dist.all_gather_object(seeds, w.seed)
        q.put((rank, got, seeds, (w.B, w.N, w.K)))
    finally:
        dist.destroy_process_group()


def _worker_fail(rank, world, port, q):
    _init(rank, world, port, timeout_s=5)
    if rank == 1:
        os._exit(3)                       # a rank that dies between steps
    try:
        bench.max_over_ranks(1.0, world, "cpu")
        q.put((rank, "no error"))
    except Exception as e:                # the surviving rank learns of it
        q.put((rank, type(e).__name__))


def _run(fn, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
    out = []
    while not q.empty():
        out.append(q.get())
    return procs, out


def test_weak_scaling_seeds_and_max_over_ranks():
    procs, out = _run(_worker_reduce, 2)
    assert all(p.exitcode == 0 for p in procs)
    assert len(out) == 2
    for rank, got, seeds, shape in out:
        assert got == 15.0                            # the slowest rank's time
        assert len(set(seeds)) == 2                   # each rank its own batch
        assert shape == (32, 32768, 2048)             # same per-rank workload


def test_failed_rank_is_detected_by_the_survivor():
    procs, out = _run(_worker_fail, 2)
    assert procs[1].exitcode == 3
    res = dict(out)
    assert 0 in res and res[0] != "no error"


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"config": 1, "steps": 1, "warmup": 0})()
    bench.run_reference(args)
    assert capsys.readouterr().out == ""
