"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2)
shard units, reduce the timed region as a max over ranks and the work as a
sum, as the NCCL ranks do on GPUs."""
import os
import socket

import pytest

from streaming_speaker_diarization_b200.dist import shard

torch = pytest.importorskip("torch")


def test_shard_covers_every_unit_once():
    for n in (0, 1, 5, 64, 65):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                lo, hi = shard(n, r, world)
                seen.extend(range(lo, hi))
            assert seen == list(range(n))
            sizes = [shard(n, r, world)[1] - shard(n, r, world)[0] for r in range(world)]
            assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from streaming_speaker_diarization_b200 import dist as sd
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = sd.shard(64, rank, world)
        ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        res = (sd.max_over_ranks(ms), sd.sum_over_ranks(hi - lo), sd.throughput(90.0, ms))
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_like_the_bench():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        mx, n, thr = got[r]
        assert mx == 15.0                            # slowest rank
        assert n == 64                               # every stream counted once
        assert abs(thr - 2 * 90.0 / 0.015) < 1e-6   # all ranks' audio / slowest time
