"""DPO with the adapter-off reference on the streamed base, on the GPU.

* sequence log-probabilities of the policy and of the reference, the loss and
  the LoRA gradients against the fp64 oracle (``oracle.train.dpo_step``);
* with every LoRA B zero the policy is the reference bit for bit, so the
  loss is exactly log 2 and d loss / d logp is +-beta / (2 P);
* streamed == resident bit for bit (loss, log-probs, every gradient).

Tolerances: the sequence log-probabilities sum S-1 bf16-derived per-token
terms (relative 1e-3, as the SFT loss).  The loss is checked twice: against
the DPO formula on the GPU's own log-probs (1e-6), and against the oracle's
loss within the bound the measured log-prob errors imply (the formula is
beta-Lipschitz in each pair's four log-probs).  Gradients 3e-2 relative
Frobenius, the whole-model bound derived in test_gpu_model.py.
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import train as OT
from test_gpu_model import model_tolerance
from tolerances import check_model_grads, rel_fro

pytestmark = pytest.mark.gpu

BETA = 0.1


def _trainer(shape, B, Sq, n_slots):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    return StreamedLoraTrainer(shape, B, Sq, n_slots=n_slots, init="host")


def _dpo(tr, ids, beta=BETA):
    tr.set_ids(ids.cuda())
    tr.forward_backward_dpo(beta)
    torch.cuda.synchronize()
    return (tr.loss_dev.item(), tr.pi_logp.double().cpu(), tr.ref_logp.double().cpu(), tr.lora.grad.clone(),
            tr.dseq.double().cpu())


@pytest.mark.parametrize("shape,B,Sq", [(S.TINY, 4, 64), (S.TINY_UNTIED, 2, 96)])
def test_dpo_matches_oracle(lsq, shape, B, Sq):
    tr = _trainer(shape, B, Sq, 2)
    ids = S.tokens(shape, B, Sq)
    loss, pi, ref, g, _ = _dpo(tr, ids)
    layers = [S.layer_weights(shape, l) for l in range(shape.n_layers)]
    emb = S.embeddings(shape)
    lora = [{n: {ab: t[ab] for ab in ("A", "B")} for n, t in per.items()} for per in S.lora_init(shape)]
    oloss, og, opi, oref = OT.dpo_step(shape, layers, emb, lora, ids, BETA)
    np.testing.assert_allclose(pi.numpy(), opi.numpy(), rtol=1e-3)
    np.testing.assert_allclose(ref.numpy(), oref.numpy(), rtol=1e-3)
    # the loss kernel computes the DPO formula on the GPU's own log-probs
    from oracle import decoder as OD
    assert abs(loss - OD.dpo_loss(pi, ref, BETA).item()) <= 1e-6 * max(1.0, abs(loss))
    # and the loss moves no more than the log-prob errors allow: |d loss| <=
    # beta * max over pairs of the summed |error| of its four log-probs (sigmoid <= 1)
    err = (pi - opi).abs() + (ref - oref).abs()
    bound = BETA * float((err[0::2] + err[1::2]).max()) + 1e-6
    assert abs(loss - oloss) <= bound, (loss, oloss, bound)
    check_model_grads(tr.lora, g, og, shape, model_tolerance(shape, B, Sq, og, dpo_beta=BETA, ids=ids),
                      what=f"dpo {shape.name}")
    tr.close()


def test_dpo_zero_b_policy_is_reference_bitwise(lsq):
    shape, B, Sq = S.TINY, 4, 64
    tr = _trainer(shape, B, Sq, 2)
    lp = tr.lora
    for l in range(shape.n_layers):
        for n in S.LINEARS:
            lp.view(lp.op, l, n, "B").zero_()
    loss, pi, ref, _, dseq = _dpo(tr, S.tokens(shape, B, Sq))
    assert torch.equal(pi, ref)
    assert abs(loss - math.log(2.0)) < 1e-6
    want = np.array([-BETA / 2 / (B // 2), BETA / 2 / (B // 2)] * (B // 2))
    np.testing.assert_allclose(dseq.numpy(), want, rtol=1e-6)
    tr.close()


def test_dpo_streamed_equals_resident_bitwise(lsq):
    shape, B, Sq = S.TINY, 2, 64
    ids = S.tokens(shape, B, Sq)
    tr_s = _trainer(shape, B, Sq, 2)
    a = _dpo(tr_s, ids)
    tr_s.close()
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    tr_r = StreamedLoraTrainer(shape, B, Sq, n_slots=None, init="host")
    b = _dpo(tr_r, ids)
    tr_r.close()
    assert a[0] == b[0]
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert torch.equal(a[3], b[3])
