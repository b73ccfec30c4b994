"""The replica bench's multi-rank host logic on CPU: two gloo ranks, each with
its own device time, agree on the slowest rank's time, and the job throughput
counts every replica's tokens against that time.  (The GPU path uses the same
functions over NCCL; replicas exchange nothing else.)"""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, q):
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(dist, times[rank], "cpu")
        value = bench.job_throughput(world, 512, 10, ms)
        dist.barrier()
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_job_throughput(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [3.5, 5.25, 4.0, 1.0][:world]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for _, ms, value in res:
        assert ms == max(times)
        assert value == pytest.approx(world * 512 * 10 / (max(times) / 1e3))


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, 2.5, "cpu") == 2.5
    assert bench.job_throughput(1, 512, 4, 2.0) == pytest.approx(512 * 4 / 2e-3)


def test_gpus_flag_starts_the_ranks_itself():
    """`bench.py --gpus 2` outside torchrun starts two ranks itself; rank 0 alone prints one line whose time is
    the slower rank's (the rank-1 time 11 ms)."""
    import json
    import subprocess
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "4",
                        "--dist-selftest"], capture_output=True, text=True, timeout=240, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["ms"] == 11.0
    assert d["value"] == pytest.approx(2 * 4 / 11e-3)


def test_gpus_flag_disagreeing_with_world_size_fails():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="3")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dist-selftest"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode != 0
