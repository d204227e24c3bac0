"""The multi-GPU path of bench.py on CPU: two gloo ranks.

Clips are independent, so N GPUs run N independent batches (weak scaling)
and the only cross-rank operations are the barrier and the max of the step
time over ranks.  These tests run those with world_size 2 on the gloo
backend, and check that a rank that never joins ends the others' wait with
an error instead of a hang."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    dist.barrier()
    m = bench.reduce_max(local_ms, dist, "cpu")
    q.put((rank, m, bench.weak_scaling_throughput(world, 368.0, m)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_take_the_max_step_time():
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
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 ranks x 368 audio-seconds per 15 ms step
    assert res[0][2] == pytest.approx(2 * 368.0 / 0.015)


def _lonely_rank(port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        dist.init_process_group("gloo", rank=0, world_size=2, timeout=datetime.timedelta(seconds=3))
        dist.barrier()
        q.put("joined")
    except Exception as e:  # the missing rank turns into an error, not a hang
        q.put(type(e).__name__)


def test_missing_rank_ends_in_an_error_not_a_hang():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_lonely_rank, args=(_free_port(), q))
    p.start()
    out = q.get(timeout=120)
    p.join(timeout=60)
    assert out != "joined"
