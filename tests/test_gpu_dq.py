"""Double-quantised absmax on the GPU, against the oracle.

* lsq_absmax_double_quantize: codes and (centre, scale) params bit for bit,
  on workload-shaped absmax arrays with ragged last blocks, constant and
  all-zero blocks, tiny centred values (E4M3 subnormals) and wide ranges;
* lsq_absmax_expand: the fp32 absmax bit for bit;
* the scheduler's expansion after an upload (several arrays per record,
  ragged sizes) bit for bit, and its argument checks;
* a training run on double-quantised records: loss and LoRA gradients
  against the oracle run on the same second-level absmax, and streamed ==
  resident bit for bit.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import nf4
from oracle import train as OT
from test_gpu_model import model_tolerance
from tolerances import check_model_grads, rel_fro

pytestmark = pytest.mark.gpu

F32 = np.float32


def _absmax_cases():
    g = np.random.default_rng(7)
    w = S.normal_f32(S.WEIGHT_SEED, 91, (5000, 64), S.BASE_STD)
    work = nf4.bf16_round(np.abs(w)).max(axis=1).astype(F32)                 # 19.5 blocks: ragged tail
    edge = np.concatenate([np.full(256, 0.0371, F32), np.zeros(256, F32),   # constant, all-zero
                           (0.05 + g.normal(0, 1e-7, 256)).astype(F32),     # tiny spread
                           g.uniform(0, 10, 256).astype(F32),               # wide spread, zeros nearby
                           np.array([0.5], F32)])                           # one-value last block
    wide = np.abs(g.standard_cauchy(3 * 256 + 100)).astype(F32)
    return [work, edge, wide]


@pytest.mark.parametrize("case", range(3))
def test_double_quantize_and_expand_bitwise(lsq, case):
    a = _absmax_cases()[case]
    nb = a.size
    nblk = (nb + 255) // 256
    d_a = torch.from_numpy(a).cuda()
    codes = torch.empty(nb, dtype=torch.uint8, device="cuda")
    params = torch.empty(nblk, 2, dtype=torch.float32, device="cuda")
    lsq.lsq_absmax_double_quantize(d_a, nb, codes, params)
    out = torch.empty(nb, dtype=torch.float32, device="cuda")
    lsq.lsq_absmax_expand(codes, params, nb, out)
    torch.cuda.synchronize()
    oc, op = nf4.double_quantize_absmax(a)
    assert np.array_equal(params.cpu().numpy().view(np.uint32), op.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), oc)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), nf4.expand_absmax(oc, op).view(np.uint32))


def test_scheduler_expands_after_upload(lsq):
    arrays = _absmax_cases()
    # record: [codes8 | params] per array; slot: record, then the fp32 outputs
    off, items, rec_parts = 0, [], []
    for a in arrays:
        c, p = nf4.double_quantize_absmax(a)
        c_off = off
        off = (off + c.size + 255) // 256 * 256
        p_off = off
        off = (off + p.nbytes + 255) // 256 * 256
        items.append([c_off, p_off, 0, a.size])
        rec_parts.append((c_off, c, p_off, p))
    rec_bytes = (off + 4095) // 4096 * 4096
    slot_bytes = rec_bytes
    for it, a in zip(items, arrays):
        it[2] = slot_bytes
        slot_bytes = (slot_bytes + 4 * a.size + 255) // 256 * 256
    host = torch.zeros(rec_bytes, dtype=torch.uint8, pin_memory=True)
    hv = host.numpy()
    for c_off, c, p_off, p in rec_parts:
        hv[c_off:c_off + c.size] = c
        hv[p_off:p_off + p.nbytes] = p.reshape(-1).view(np.uint8)
    slots = [torch.full((slot_bytes,), 0xFF, dtype=torch.uint8, device="cuda") for _ in range(2)]
    copy = torch.cuda.Stream()
    st = lsq.lsq_stream_create(1, 2, rec_bytes, [s.data_ptr() for s in slots], [host.data_ptr()],
                               torch.cuda.current_stream(), copy)
    try:
        bad = [list(items[0])]
        bad[0][2] = rec_bytes - 256                                     # output overlaps the record
        with pytest.raises(lsq.LsqError) as e:
            lsq.lsq_stream_set_absmax_expand(st, [tuple(x) for x in bad], slot_bytes)
        assert e.value.status == 1
        with pytest.raises(lsq.LsqError):
            lsq.lsq_stream_set_absmax_expand(st, [tuple(items[0])], 4 * arrays[0].size - 4 + rec_bytes)
        lsq.lsq_stream_set_absmax_expand(st, [tuple(x) for x in items], slot_bytes)
        lsq.lsq_layer_upload_async(st, 0, 1)
        copy.synchronize()
        with pytest.raises(lsq.LsqError) as e:                          # too late: an upload happened
            lsq.lsq_stream_set_absmax_expand(st, [tuple(x) for x in items], slot_bytes)
        assert e.value.status == 5
        got = slots[1].cpu().numpy()
        for it, a in zip(items, arrays):
            want = nf4.double_quantized(a).view(np.uint8)
            assert np.array_equal(got[it[2]:it[2] + 4 * a.size], want)
        assert np.all(slots[0].cpu().numpy() == 0xFF)                   # the other slot untouched
    finally:
        lsq.lsq_stream_destroy(st)


def _trainer(shape, B, Sq, n_slots, init="host"):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    return StreamedLoraTrainer(shape, B, Sq, n_slots=n_slots, init=init, absmax="dq8")


def _run(tr, shape, B, Sq, steps):
    losses, grads0 = [], None
    for t in range(steps):
        tr.set_ids(S.tokens(shape, B, Sq, step=t).cuda())
        tr.forward_backward()
        torch.cuda.synchronize()
        losses.append(tr.loss_dev.item())
        if t == 0:
            grads0 = tr.lora.grad.clone()
        tr.optimizer_step()
    torch.cuda.synchronize()
    return losses, grads0


def test_dq_model_matches_oracle(lsq):
    shape, B, Sq, steps = S.TINY_UNTIED, 1, 200, 2
    tr = _trainer(shape, B, Sq, 2)
    assert tr.layout.nbytes < tr.layout.slot_bytes
    losses, g0 = _run(tr, shape, B, Sq, steps)
    layers = [S.layer_weights(shape, l) for l in range(shape.n_layers)]
    lora = [{n: {ab: t[ab] for ab in ("A", "B")} for n, t in per.items()} for per in S.lora_init(shape)]
    ids = [S.tokens(shape, B, Sq, step=t) for t in range(steps)]
    ol, og, _ = OT.train(shape, layers, S.embeddings(shape), lora, ids, double_quant=True)
    for a, b in zip(losses, ol):
        assert abs(a - b) <= 1e-3 * abs(b), (losses, ol)
    check_model_grads(tr.lora, g0, og, shape, model_tolerance(shape, B, Sq, og, double_quant=True),
                      what=f"dq8 {shape.name}")
    tr.close()


def test_dq_streamed_equals_resident_bitwise(lsq):
    shape, B, Sq, steps = S.TINY_UNTIED, 2, 128, 3
    ref = _trainer(shape, B, Sq, None, init="device")
    rl, rg = _run(ref, shape, B, Sq, steps)
    ref.close()
    tr = _trainer(shape, B, Sq, 2, init="device")
    sl, sg = _run(tr, shape, B, Sq, steps)
    uploads, nbytes, _ = tr.stats()
    tr.close()
    assert sl == rl and torch.equal(sg, rg)
    assert nbytes == uploads * tr.layout.nbytes          # only the 8-bit records crossed the link
