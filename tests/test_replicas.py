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


def test_gpus_flag_launches_one_rank_per_gpu():
    """`bench.py --gpus 2` without WORLD_SIZE re-runs itself as two ranks
    (torch.distributed.run, rendezvous on 127.0.0.1); the line reports both."""
    import json
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                          "--steps", "5", "--dry-run"], env=env, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["gpus_flag"] == 2
    assert line["ms_per_step"] == pytest.approx(11.0 / 5)   # the slower rank's time
    assert line["value"] == pytest.approx(4 * 2 * 5 / 0.011)


def test_gpus_flag_must_match_the_launch():
    import subprocess
    import sys
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                          "--dry-run"], env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode == 2 and "WORLD_SIZE=3" in out.stderr
