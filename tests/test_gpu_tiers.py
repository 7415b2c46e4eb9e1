"""The disk tier and the host-resident embedding, on the GPU.

* records read from a store file by the library's reader threads (through
  page-locked staging buffers and the copy stream's bounded host waits) train
  bit-identically to records held in page-locked RAM - also with
  double-quantised absmax;
* a store file shorter than the records it must hold is refused at creation;
* an untied embedding gathered straight from page-locked host RAM (zero-copy)
  trains bit-identically to one held in HBM;
* the lm_head in page-locked host RAM, streamed in vocabulary chunks through
  two HBM buffers, trains bit-identically to the resident head.
"""
import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu


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


@pytest.mark.parametrize("absmax", ["fp32", "dq8"])
def test_disk_tier_equals_ram_bitwise(lsq, tmp_path, absmax):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    shape, B, Sq, steps = S.TINY_UNTIED, 2, 128, 3
    ram = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device", absmax=absmax)
    rl, rg = _run(ram, shape, B, Sq, steps)
    rstats = ram.stats()
    ram.close()
    path = str(tmp_path / "store.bin")
    disk = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device", absmax=absmax, source="disk",
                               store_path=path)
    assert disk.host_records == []                         # nothing of the base stays in RAM
    dl, dg = _run(disk, shape, B, Sq, steps)
    dstats = disk.stats()
    disk.close()
    assert dl == rl and torch.equal(dg, rg)
    assert dstats == rstats


def test_short_store_file_is_refused(lsq, tmp_path):
    path = tmp_path / "short.bin"
    path.write_bytes(b"\0" * (3 << 16))                    # 3 parts of 64 KiB, 4 needed
    slots = [torch.empty(1 << 16, dtype=torch.uint8, device="cuda") for _ in range(2)]
    staging = [torch.empty(1 << 16, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
    with pytest.raises(lsq.LsqError) as e:
        lsq.lsq_stream_create(4, 2, 1 << 16, [s.data_ptr() for s in slots], None, torch.cuda.current_stream(),
                              torch.cuda.Stream(), disk=(str(path), [b.data_ptr() for b in staging], 2))
    assert e.value.status == 1
    pageable = [torch.empty(1 << 16, dtype=torch.uint8) for _ in range(2)]
    path.write_bytes(b"\0" * (4 << 16))
    with pytest.raises(lsq.LsqError) as e:
        lsq.lsq_stream_create(4, 2, 1 << 16, [s.data_ptr() for s in slots], None, torch.cuda.current_stream(),
                              torch.cuda.Stream(), disk=(str(path), [b.data_ptr() for b in pageable], 2))
    assert e.value.status == 2


def test_disk_tier_reads_every_byte(lsq, tmp_path):
    """Scheduler alone: 5 layer parts of odd content through 2 staging buffers and 3 reader
    threads (slices of unequal length), uploaded in the policy's order; each slot checked."""
    import numpy as np
    n_layers, nbytes = 5, 3 * 4096 + 256
    recs = [np.random.default_rng(l).integers(0, 256, nbytes, dtype=np.uint8) for l in range(n_layers)]
    path = tmp_path / "parts.bin"
    path.write_bytes(b"".join(r.tobytes() for r in recs))
    slots = [torch.zeros(nbytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    staging = [torch.empty(nbytes, dtype=torch.uint8, pin_memory=True) for _ in range(2)]
    copy = torch.cuda.Stream()
    st = lsq.lsq_stream_create(n_layers, 2, nbytes, [s.data_ptr() for s in slots], None,
                               torch.cuda.current_stream(), copy, disk=(str(path), [b.data_ptr() for b in staging], 3))
    try:
        for l in list(range(n_layers)) + list(reversed(range(n_layers))):
            ptr = lsq.lsq_stream_step(st, l, 1)
            slot = [s.data_ptr() for s in slots].index(ptr)
            torch.cuda.current_stream().synchronize()
            assert np.array_equal(slots[slot].cpu().numpy(), recs[l]), l
    finally:
        torch.cuda.synchronize()
        lsq.lsq_stream_destroy(st)


def test_host_embedding_equals_hbm_bitwise(lsq):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    shape, B, Sq, steps = S.TINY_UNTIED, 2, 128, 2
    a = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device")
    al, ag = _run(a, shape, B, Sq, steps)
    a.close()
    b = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device", embed="host")
    assert not b.embed.is_cuda and b.embed.is_pinned()
    bl, bg = _run(b, shape, B, Sq, steps)
    b.close()
    assert al == bl and torch.equal(ag, bg)
    with pytest.raises(ValueError):
        StreamedLoraTrainer(S.TINY, 1, 64, n_slots=2, init="device", embed="host")   # tied: lm_head needs it


@pytest.mark.parametrize("shape,B,Sq", [(S.TINY_UNTIED, 2, 128), (S.TINY, 2, 96)])
def test_streamed_head_equals_resident_bitwise(lsq, shape, B, Sq):
    """The lm_head in page-locked host RAM, streamed in vocabulary chunks (256
    rows: 4 chunks with a ragged last one of 232 rows for the untied 1000-row
    head, 2 for the tied 512-row table, which then also serves the gather),
    trains bit-identically to the resident head: logits, loss curve,
    gradients; also the DPO step, which runs the head three times."""
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    steps = 3
    a = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device")
    al, ag = _run(a, shape, B, Sq, steps)
    alog = a.logits.clone()
    a.set_ids(S.tokens(shape, B, Sq, step=9).cuda())
    a.forward_backward_dpo(0.1)
    adpo = (a.loss_dev.clone(), a.lora.grad.clone())
    a.close()
    b = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device", head="host", head_chunk=256)
    assert not b.lm_head.is_cuda and b.lm_head.is_pinned()
    assert b.embed.is_cuda != shape.tied
    bl, bg = _run(b, shape, B, Sq, steps)
    blog = b.logits.clone()
    b.set_ids(S.tokens(shape, B, Sq, step=9).cuda())
    b.forward_backward_dpo(0.1)
    bdpo = (b.loss_dev.clone(), b.lora.grad.clone())
    uploads, nbytes, _ = b.head_stats()
    b.close()
    n_chunks = -(-shape.vocab // 256)
    # every pass over the head walks its chunks in order; more chunks than the two buffers means
    # each pass uploads all of them (2 per training step, 3 for the DPO step), else they stay
    passes = 2 * steps + 3
    assert uploads == (passes * n_chunks if n_chunks > 2 else n_chunks), uploads
    assert nbytes == uploads * 256 * shape.d * 2
    assert al == bl and torch.equal(ag, bg) and torch.equal(alog, blog)
    assert torch.equal(adpo[0], bdpo[0]) and torch.equal(adpo[1], bdpo[1])
