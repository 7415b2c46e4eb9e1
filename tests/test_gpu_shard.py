"""Sharded upload on one GPU (the only multi-GPU-free form of it).

With a one-rank NCCL group the scheduler still runs the whole path: this
rank's part of each record (all of it), the gather callback on the copy
stream (an in-place NCCL all-gather), then the upload's event.  Training
through it must equal the plain streamed run bit for bit, and a failing
callback must surface as LSQ_ECALLBACK.  The two-rank reassembly is covered
on CPU (tests/test_dist_cpu.py).
"""
import datetime
import socket

import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.fixture
def one_rank_group():
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


def _run(tr, shape, B, Sq, steps):
    losses = []
    for t in range(steps):
        tr.set_ids(S.tokens(shape, B, Sq, step=t).cuda())
        tr.forward_backward()
        torch.cuda.synchronize()
        losses.append(tr.loss_dev.item())
        if t == 0:
            g0 = tr.lora.grad.clone()
        tr.optimizer_step()
    torch.cuda.synchronize()
    return losses, g0


def test_sharded_upload_one_rank_equals_plain_bitwise(lsq, one_rank_group):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    shape, B, Sq, steps = S.TINY_UNTIED, 2, 128, 3
    plain = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device")
    pl, pg = _run(plain, shape, B, Sq, steps)
    plain.close()
    for absmax in ("fp32", "dq8"):
        tr = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device", shard=(0, 1), absmax=absmax)
        calls = []
        inner = tr._gather
        tr._gather = lambda *a: (calls.append(a[0]), inner(*a))[1]
        sl, sg = _run(tr, shape, B, Sq, steps)
        uploads, nbytes, _ = tr.stats()
        tr.close()
        assert len(calls) == uploads > shape.n_layers
        if absmax == "fp32":
            assert sl == pl and torch.equal(sg, pg)


def test_failing_gather_is_reported(lsq):
    rec = torch.zeros(1 << 16, dtype=torch.uint8, pin_memory=True)
    slots = [torch.empty(1 << 16, dtype=torch.uint8, device="cuda") for _ in range(2)]

    def bad(*_):
        raise RuntimeError("peer gone")
    copy = torch.cuda.Stream()
    st = lsq.lsq_stream_create(1, 2, 1 << 16, [s.data_ptr() for s in slots], [rec.data_ptr()],
                               torch.cuda.current_stream(), copy, shard=(0, 1, bad))
    try:
        with pytest.raises(lsq.LsqError) as e:
            lsq.lsq_layer_upload_async(st, 0, 0)
        assert e.value.status == 7
    finally:
        copy.synchronize()
        lsq.lsq_stream_destroy(st)


def test_shard_arguments_are_checked(lsq):
    rec = torch.zeros(1 << 16, dtype=torch.uint8, pin_memory=True)
    slots = [torch.empty(1 << 16, dtype=torch.uint8, device="cuda") for _ in range(2)]
    args = (1, 2, 1 << 16, [s.data_ptr() for s in slots], [rec.data_ptr()], torch.cuda.current_stream(),
            torch.cuda.Stream())
    for shard in ((2, 2, lambda *_: None), (0, 3, lambda *_: None)):   # rank out of range; 65536 % (256 * 3)
        with pytest.raises(lsq.LsqError) as e:
            lsq.lsq_stream_create(*args, shard=shard)
        assert e.value.status == 1
