"""The multi-GPU path of the benchmark on the CPU: the layer has no exchange
step, so N GPUs run N independent replicas and the only collectives are the
barrier and the max-over-ranks of the device time.  These tests run those
host-side pieces as two `gloo` ranks (no GPU needed)."""
import argparse
import datetime
import multiprocessing as mp
import os
import socket

import pytest

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        r, lr, w = bench.env_rank()
        dist.barrier()
        # rank-dependent device times: the job's time is the slowest replica's
        ms = bench.max_over_ranks(40.0 + 10.0 * rank, dist, "cpu")
        value = bench.job_rate(4, w, 100, ms)
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, r, lr, w, ms, value, None))
    except Exception as e:  # reported to the parent instead of hanging it
        q.put((rank, None, None, None, None, None, repr(e)))


def test_two_replicas_agree_on_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for rank, (r, r_env, lr, w, ms, value, err) in enumerate(got):
        assert err is None, err
        assert (r, r_env, lr, w) == (rank, rank, rank, world)
        assert ms == 50.0                      # max over the two ranks
        assert value == pytest.approx(4 * 2 * 100 / 0.050)  # units of all ranks / job time
    assert all(p.exitcode == 0 for p in procs)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.job_rate(4, 1, 200, 11.0) == pytest.approx(4 * 200 / 0.011)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(argparse.Namespace(steps=1, warmup=0)) == 0
    assert capsys.readouterr().out == ""


def test_packed_buffers_are_aligned_and_disjoint():
    offs, total = bench._packed([("a", 10), ("b", 256), ("c", 1), ("d", 0), ("e", 300)])
    assert all(o % 256 == 0 for o in offs.values())
    assert offs == {"a": 0, "b": 256, "c": 512, "d": 768, "e": 768}
    assert total == 768 + 512
