"""Data-parallel host logic on CPU with gloo, world size 2: gradient averaging
and max-over-ranks timing, as bench.py uses them under torchrun."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from nf4_layer_streamed_blockwise_b200 import dist as D
    import torch.distributed as dist
    r, w, _ = D.init_from_env(backend="gloo", timeout_s=60)
    g = torch.arange(10, dtype=torch.float32) * (r + 1)          # rank-specific gradient
    D.average_gradients(g, w)
    t = D.max_over_ranks(1.5 + r, w)
    out[rank] = (g.tolist(), t)
    dist.barrier()
    dist.destroy_process_group()


def test_gradient_mean_and_max_time_two_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    want = [i * 1.5 for i in range(10)]                          # mean of 1x and 2x
    for r in range(world):
        g, t = out[r]
        assert g == pytest.approx(want)
        assert t == 2.5
