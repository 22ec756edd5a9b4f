"""The multi-rank host logic of bench.py on CPU: two gloo ranks reduce their
timings to the max, aggregate bytes over ranks, draw distinct data, and the
reference arm does no work on ranks other than 0."""

import os
import socket
import subprocess
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


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 5.0 * (2 - rank), 1.0]
        got = bench.max_over_ranks(local, dist, "cpu")
        dist.barrier()
        q.put((rank, got, bench.rank_seed(rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    for _, got, _ in results:
        assert got == [11.0, 10.0, 1.0]
    assert results[0][2] != results[1][2]


def test_aggregate_is_weak_scaled():
    sys.path.insert(0, ROOT)
    import bench

    one = bench.aggregate_gbs(1e9, 10, 100.0, 1)
    two = bench.aggregate_gbs(1e9, 10, 100.0, 2)
    assert one == pytest.approx(100.0) and two == pytest.approx(200.0)


def test_reference_arm_is_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
