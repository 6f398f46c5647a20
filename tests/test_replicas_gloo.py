"""Multi-process host logic (world size 2, gloo on CPU): the max-over-ranks timing used for
multi-GPU numbers, and clip sharding that covers every clip exactly once."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from encoder_free_audio_b200 import replicas, synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local = [1.25, 3.5][rank]
    m = replicas.max_over_ranks(local, world)
    dist.barrier()
    so = synth.offsets_from_lengths([16000 * (1 + (i % 7)) for i in range(37)])
    c0, c1, sub = replicas.shard_clips(so, rank, world)
    q.put((rank, m, c0, c1, int(sub[-1])))
    dist.destroy_process_group()


def test_max_over_ranks_and_sharding_two_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[1] for g in got] == [3.5, 3.5]  # every rank sees the slowest rank's time
    # the shares tile the clip range in order
    assert got[0][2] == 0 and got[0][3] == got[1][2] and got[1][3] == 37


def test_shard_clips_balanced_and_exhaustive():
    so = synth.offsets_from_lengths(np.random.default_rng(3).integers(800, 480000, 200))
    for world in (1, 2, 3, 8):
        covered = []
        frames = []
        for r in range(world):
            c0, c1, sub = replicas.shard_clips(so, r, world)
            covered += list(range(c0, c1))
            frames.append(int(((sub[1:] - sub[:-1]) // 800).sum()))
            assert sub[0] == 0
        assert covered == list(range(200))
        total = int(((so[1:] - so[:-1]) // 800).sum())
        assert sum(frames) == total
        assert max(frames) - min(frames) <= 2 * 600  # each share boundary is off by at most one clip (<= 600 frames)


def test_job_throughput():
    assert replicas.job_throughput([12800, 12800], 0.5) == 51200.0
