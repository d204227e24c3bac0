"""One long clip split over ranks (audio_encoder_b200.shard), host side.

The ranges must tile the clip in whole 800-frame chunks, and the maximum of
the per-range log-mel maxima (here from the oracle, exchanged by two gloo
ranks with a max all-reduce, the one collective the split needs) must be the
whole clip's maximum, which every range is then encoded against."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from audio_encoder_b200 import shard

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("n", [0, 1, 159, 128000, 128001, 300000, 1_024_000, 9_600_000, 57_600_000])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_ranges_tile_the_clip_in_whole_chunks(n, world):
    rs = shard.chunk_ranges(n, world)
    assert len(rs) == world
    assert rs[0][0] == 0 and rs[-1][1] == n
    for (b0, e0), (b1, e1) in zip(rs, rs[1:]):
        assert e0 == b1
    sizes = []
    for b, e in rs:
        assert b <= e
        if e > b:
            assert b % shard.CHUNK_SAMPLES == 0
            assert e == n or e % shard.CHUNK_SAMPLES == 0
        sizes.append(-(-(e - b) // shard.CHUNK_SAMPLES))
    assert max(sizes) - min(sizes) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, n, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from audio_encoder_b200 import shard, synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    pcm = synth.pcm_long(3, n)
    b, e = shard.chunk_ranges(n, world)[rank]
    f0, f1 = b // 160, (n // 160 if e == n else e // 160)
    local = float(oracle.logmel_raw(pcm, f0, f1).max()) if f1 > f0 else float("-inf")
    t = torch.tensor([local], dtype=torch.float32)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    q.put((rank, local, float(t.item())))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_agree_on_the_whole_clip_maximum():
    import oracle
    from audio_encoder_b200 import synth
    n = 2 * 128000 + 48000  # three chunks, the last one partial: ranks take 2 and 1
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, n, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    whole = float(np.float32(oracle.clip_log_max(synth.pcm_long(3, n))))
    assert res[0][2] == res[1][2] == pytest.approx(whole, abs=1e-6)
    assert max(res[0][1], res[1][1]) == res[0][2]
