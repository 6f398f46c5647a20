"""Failure detection without a GPU fault.

On the GPU, a pipeline wait that can never be satisfied gives up after its poll limit, records
DMEL_DEVERR_WAIT_TIMEOUT in the device error word and returns; the context stays usable. On the
host, a rank that fails before the timing collective makes the other rank's collective end with
an error (short process-group timeout) instead of waiting for ever."""
import os
import socket

import pytest
import torch.multiprocessing as mp


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_survives():
    import torch
    from encoder_free_audio_b200 import build, dmel
    build.build()
    dmel.dmel_get_device_error(clear=True)
    bits = dmel.dmel_debug_wait_timeout(1 << 14)
    assert bits & dmel.DMEL_DEVERR_WAIT_TIMEOUT
    # the context still runs work afterwards
    codes = torch.zeros((10, 80), dtype=torch.uint8, device="cuda:0")
    T = torch.ones((1280, 256), dtype=torch.float32, device="cuda:0")
    out = torch.empty((10, 256), dtype=torch.float32, device="cuda:0")
    dmel.dmel_embed(codes, T, out)
    torch.cuda.synchronize()
    assert torch.all(out == 80.0)
    assert dmel.dmel_get_device_error(clear=True) == 0


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, port, q):
    from datetime import timedelta
    import torch.distributed as dist
    from encoder_free_audio_b200 import replicas
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=2, timeout=timedelta(seconds=5))
    if rank == 1:
        q.put((1, "raised"))
        raise RuntimeError("rank 1 fails before the timing collective")
    try:
        replicas.max_over_ranks(1.0, 2)
        q.put((0, "returned"))
    except Exception as e:  # the collective must end with an error, not hang
        q.put((0, "error: " + type(e).__name__))


def test_failed_rank_ends_the_collective_with_an_error():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_rank, args=(r, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(60)
    alive = [p.is_alive() for p in ps]
    for p in ps:
        if p.is_alive():
            p.kill()
    assert not any(alive), "a rank hung"
    got = dict(q.get(timeout=5) for _ in range(2))
    assert got[1] == "raised"
    assert got[0].startswith("error"), got[0]
