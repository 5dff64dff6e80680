"""Multi-rank host logic of bench.py on CPU: two gloo ranks, no GPU.

The BitLinear path has no exchange step, so N GPUs run independent replicas;
what is shared is the timing protocol: a barrier on both sides, the slowest
rank's time, and the units of every rank over that time."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    bench.barrier()
    mx = bench.reduce_max(1.5 + rank)  # rank 1 is the slower one
    val = bench.aggregate(1000.0, steps=10, world=world, max_seconds=mx)
    bench.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, val))


def test_two_rank_max_time_and_aggregate():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]              # both ranks see the slowest time
    assert res[0][2] == pytest.approx(1000.0 * 10 * 2 / 2.5)


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                          "--warmup", "3", "--gpus", "2"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""
