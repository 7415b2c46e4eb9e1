"""Whole-model streamed NF4-LoRA training on the GPU.

* per-step loss against the fp64 oracle within 1e-3 relative (whole-model
  configurations), LoRA gradients within the tolerance below;
* streamed == resident bit for bit: logits, every LoRA gradient and a 5-step
  loss curve, for several slot counts (the pages' regression test: a
  streamed run feeds identical quantised bytes to identical kernels);
* the first layer's LoRA gradients are not zero (the pages' other streaming
  regression check);
* a pageable store is refused, and the first upload into a slot lands after
  compute-stream work still queued on the slot's recycled memory.

Gradient tolerance: the GPU keeps activations and their gradients in bf16
between kernels (as the pages' bf16 trainer does) while the oracle is fp64
end to end, and the LoRA gradients are sensitive to that storage rounding
(0.5% to 3% relative Frobenius error per tensor).  bf16_model.py models it
(the oracle's own forward and backward with bf16 rounding at the kernels'
storage points); each tensor is held to twice that model's error against the
oracle, never tighter than 5e-3.
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import train as OT
import bf16_model as BM
from tolerances import check_model_grads, record, rel_fro

pytestmark = pytest.mark.gpu



def _trainer(shape, B, Sq, n_slots, init="host"):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    return StreamedLoraTrainer(shape, B, Sq, n_slots=n_slots, init=init)


def _run(tr, shape, B, Sq, steps):
    losses = []
    grads0 = None
    for t in range(steps):
        tr.set_ids(S.tokens(shape, B, Sq, step=t).cuda())
        tr.forward_backward()
        torch.cuda.synchronize()
        losses.append(tr.loss_dev.item())
        if t == 0:
            grads0 = tr.lora.grad.clone()
            logits0 = tr.logits.clone()
        tr.optimizer_step()
    torch.cuda.synchronize()
    return losses, grads0, logits0


def _check_losses(losses, ref, what):
    for t, (a, b) in enumerate(zip(losses, ref)):
        record(f"{what} loss step {t}", "loss", rel=abs(a - b) / abs(b), rel_bound=1e-3)
        assert abs(a - b) <= 1e-3 * abs(b), (losses, ref)


def model_tolerance(shape, B, Sq, ref_grads, double_quant=False, dpo_beta=None, ids=None):
    """Per-tensor gradient tolerance from the bf16 storage model (bf16_model.tolerance) on the
    first step's inputs."""
    from oracle import train as OT
    layers = [OT.dequantized_layer(S.layer_weights(shape, l), double_quant) for l in range(shape.n_layers)]
    emb = {k: v.to(torch.float64) for k, v in S.embeddings(shape).items()}
    ops = [{n: {ab: OT.operand(t[ab]) for ab in ("A", "B")} for n, t in per.items()} for per in S.lora_init(shape)]
    ids = S.tokens(shape, B, Sq, step=0) if ids is None else ids
    if dpo_beta is None:
        mg = BM.sft_grads(ids, layers, emb, ops, shape)
    else:
        mg = BM.dpo_grads(ids, layers, emb, ops, shape, dpo_beta)
    return BM.tolerance(ref_grads, mg)


def _oracle(shape, B, Sq, steps):
    layers = [S.layer_weights(shape, l) for l in range(shape.n_layers)]
    emb = S.embeddings(shape)
    lora = [{n: {ab: t[ab] for ab in ("A", "B")} for n, t in per.items()} for per in S.lora_init(shape)]
    ids = [S.tokens(shape, B, Sq, step=t) for t in range(steps)]
    return OT.train(shape, layers, emb, lora, ids)


@pytest.mark.parametrize("shape,B,Sq", [(S.TINY, 2, 128), (S.TINY_UNTIED, 1, 200)])
def test_model_matches_oracle(lsq, shape, B, Sq):
    steps = 3
    tr = _trainer(shape, B, Sq, 2)
    losses, g0, _ = _run(tr, shape, B, Sq, steps)
    ol, og, _ = _oracle(shape, B, Sq, steps)
    _check_losses(losses, ol, shape.name)
    check_model_grads(tr.lora, g0, og, shape, model_tolerance(shape, B, Sq, og), what=shape.name)
    tr.close()


def test_smollm2_shape_loss_matches_oracle(lsq):
    shape, B, Sq, steps = S.SMOL, 1, 512, 2
    tr = _trainer(shape, B, Sq, 2)
    losses, g0, _ = _run(tr, shape, B, Sq, steps)
    ol, og, _ = _oracle(shape, B, Sq, steps)
    _check_losses(losses, ol, shape.name)
    check_model_grads(tr.lora, g0, og, shape, model_tolerance(shape, B, Sq, og), what=shape.name)
    tr.close()


@pytest.mark.parametrize("shape,B,Sq", [(S.TINY_UNTIED, 2, 128), (S.SMOL, 1, 512)])
def test_streamed_equals_resident_bitwise(lsq, shape, B, Sq):
    steps = 5
    ref = _trainer(shape, B, Sq, None, init="device")
    rl, rg, rlog = _run(ref, shape, B, Sq, steps)
    up, _, _ = ref.stats()
    assert up == shape.n_layers            # resident: every layer uploaded once
    ref.close()
    for n_slots in (2, 3, 8):
        tr = _trainer(shape, B, Sq, n_slots, init="device")
        sl, sg, slog = _run(tr, shape, B, Sq, steps)
        uploads, nbytes, reused = tr.stats()
        tr.close()
        assert sl == rl, (n_slots, sl, rl)
        assert torch.equal(sg, rg), n_slots
        assert torch.equal(slog, rlog), n_slots
        if n_slots < shape.n_layers:
            assert uploads > shape.n_layers     # the backward re-streamed layers
        assert reused >= 1                       # the turnaround layer was not re-uploaded


def test_unpinned_store_is_rejected(lsq):
    t = torch.empty(1 << 20, dtype=torch.uint8)          # pageable
    slots = [torch.empty(1 << 20, dtype=torch.uint8, device="cuda") for _ in range(2)]
    with pytest.raises(lsq.LsqError) as e:
        lsq.lsq_stream_create(1, 2, 1 << 20, [s.data_ptr() for s in slots], [t.data_ptr()],
                              torch.cuda.current_stream(), torch.cuda.Stream())
    assert e.value.status == 2


def test_first_upload_waits_for_queued_compute_work(lsq):
    """The allocator may hand out a slot's memory while a kernel that writes
    the block's previous tensor is still queued on the compute stream; the
    first upload into the slot must land after it (the scheduler orders it
    behind the compute stream's work at creation)."""
    nbytes = 64 << 20
    g = torch.Generator().manual_seed(5)
    rec = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, generator=g).pin_memory()
    compute, copy = torch.cuda.current_stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    junk = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    ptr = junk.data_ptr()
    torch.cuda._sleep(100_000_000)       # about 50 ms of compute-stream work ahead of ...
    junk.fill_(7)                        # ... a write into the block
    del junk
    slots = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    assert slots[0].data_ptr() == ptr    # the block was recycled with the write still queued
    st = lsq.lsq_stream_create(1, 2, nbytes, [s.data_ptr() for s in slots], [rec.data_ptr()], compute, copy)
    try:
        lsq.lsq_layer_upload_async(st, 0, 0)
        torch.cuda.synchronize()
        assert torch.equal(slots[0].cpu(), rec)
    finally:
        lsq.lsq_stream_destroy(st)
