"""The bf16 storage model behind the whole-model gradient tolerance
(bf16_model.py), on the CPU: with its roundings switched off it is the oracle
(same loss gradients to 1e-12), and with them on it moves the LoRA gradients
by the fraction of a percent to few percent that the GPU shows, far below
what a kernel mistake would."""
import numpy as np
import torch

import bf16_model as BM
import synthetic as S
from oracle import decoder as D
from oracle import train as OT


def _inputs(shape, B, Sq):
    layers = [OT.dequantized_layer(S.layer_weights(shape, l)) for l in range(shape.n_layers)]
    emb = {k: v.to(torch.float64) for k, v in S.embeddings(shape).items()}
    ops = [{n: {ab: OT.operand(t[ab]) for ab in ("A", "B")} for n, t in per.items()} for per in S.lora_init(shape)]
    return S.tokens(shape, B, Sq, step=0), layers, emb, ops


def _rf(a, b):
    return float(torch.linalg.norm(a - b) / torch.linalg.norm(b))


def test_storage_model_without_rounding_is_the_oracle_and_with_it_moves_gradients_by_percents():
    shape, B, Sq = S.TINY, 1, 64
    ids, layers, emb, ops = _inputs(shape, B, Sq)
    _, ref = D.model_loss_and_grads(ids, layers, emb, ops, shape)
    BM.ROUNDING[0] = False
    try:
        plain = BM.sft_grads(ids, layers, emb, ops, shape)
    finally:
        BM.ROUNDING[0] = True
    stored = BM.sft_grads(ids, layers, emb, ops, shape)
    errs = []
    for l in range(shape.n_layers):
        for n in S.LINEARS:
            for ab in ("A", "B"):
                assert _rf(plain[l][n][ab], ref[l][n][ab]) < 1e-12
                errs.append(_rf(stored[l][n][ab], ref[l][n][ab]))
    assert 1e-3 < float(np.median(errs)) and max(errs) < 5e-2, errs
    tol = BM.tolerance(ref, stored)
    assert min(tol.values()) >= 5e-3 and max(tol.values()) < 0.1


def test_tolerance_catches_a_planted_mistake():
    """A plausible slip in the computation (RoPE at the wrong base, here the
    8B stack's theta on the tiny stack) moves the LoRA gradients far outside
    the tolerance."""
    import dataclasses
    shape, B, Sq = S.TINY, 1, 64
    ids, layers, emb, ops = _inputs(shape, B, Sq)
    _, ref = D.model_loss_and_grads(ids, layers, emb, ops, shape)
    tol = BM.tolerance(ref, BM.sft_grads(ids, layers, emb, ops, shape))
    wrong = dataclasses.replace(shape, theta=5e5)
    _, bad = D.model_loss_and_grads(ids, layers, emb, ops, wrong)
    outside = [_rf(bad[l][n][ab], ref[l][n][ab]) > tol[(l, n, ab)]
               for l in range(shape.n_layers) for n in ("q", "k") for ab in ("A", "B")]
    assert all(outside)
