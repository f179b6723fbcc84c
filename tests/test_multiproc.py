"""Host logic of the multi-GPU benchmark on CPU ranks (gloo, world size 2):
the slowest rank's time reaches every rank, the whole-job value counts the
work of all ranks, every rank draws its own inputs (weak scaling with no
data-path collective), and the reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 2.0 + rank  # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, dist, "cpu")
        value = bench.whole_job(9_191_424 * 16, world, slowest) / 1e9
        q.put((rank, slowest, value, bench.replica_seed(rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_share_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [3.0, 3.0]           # max over ranks, on every rank
    assert res[0][2] == pytest.approx(2 * 9_191_424 * 16 / 3e-3 / 1e9)
    assert res[0][3] != res[1][3]                        # independent inputs per rank


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(1.25, None) == 1.25
    assert bench.whole_job(100, 1, 1.0) == pytest.approx(1e5)


def test_reference_arm_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0
    assert out.stdout.strip() == ""
