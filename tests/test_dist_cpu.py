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


def _shard_worker(rank, world, port, out):
    """Sharded upload on CPU: every rank holds 1/world of each layer record; the
    uploads follow the scheduler's own policy (lsq_stream_simulate) for a
    forward + backward walk, each followed by the all-gather the trainer runs;
    at every compute wait the slot must hold the whole record."""
    import numpy as np
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from nf4_layer_streamed_blockwise_b200 import dist as D
    from nf4_layer_streamed_blockwise_b200 import lib as L
    import torch.distributed as dist
    r, w, _ = D.init_from_env(backend="gloo", timeout_s=60)
    n_layers, n_slots, nbytes = 6, 3, 256 * w * 5
    records = [torch.from_numpy(np.random.default_rng(100 + l).integers(0, 256, nbytes, dtype=np.uint8))
               for l in range(n_layers)]
    lo, hi = D.shard_range(nbytes, r, w)
    host = [rec[lo:hi].clone() for rec in records]            # all this rank keeps of the base
    slots = [torch.full((nbytes + 64,), 7, dtype=torch.uint8) for _ in range(n_slots)]
    steps = [(l, 1) for l in range(n_layers)] + [(l, -1) for l in reversed(range(n_layers))]
    acts = L.lsq_stream_simulate(n_layers, n_slots, steps)
    ok, uploads = True, 0
    held = {}
    for kind, layer, slot in acts:
        if kind == 2:                                           # upload: own part, then the gather
            slots[slot][lo:hi].copy_(host[layer])
            D.gather_slot(slots[slot], nbytes, r, w)
            held[slot] = layer
            uploads += 1
        elif kind == 3:                                         # compute waits for the layer
            ok &= held.get(slot) == layer and torch.equal(slots[slot][:nbytes], records[layer])
            ok &= bool((slots[slot][nbytes:] == 7).all())
    out[rank] = (ok, uploads, acts)
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_upload_reassembles_every_record_two_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][0] and out[1][0]
    assert out[0][2] == out[1][2]            # same uploads in the same order: the collectives pair up
    assert out[0][1] > 6                     # the backward re-streamed layers


def test_shard_range_partitions_the_record():
    from nf4_layer_streamed_blockwise_b200 import dist as D
    for world in (1, 2, 3, 8):
        n = 4096 * world
        parts = [D.shard_range(n, r, world) for r in range(world)]
        assert parts[0][0] == 0 and parts[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
    with pytest.raises(ValueError):
        D.shard_range(1000, 0, 3)
