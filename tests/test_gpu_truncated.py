"""Whole-model training at full width on truncated stacks.

The Qwen2.5-3B and Llama-3.1-8B shapes at their real widths (hidden 2048 /
4096, SwiGLU 11008 / 14336, 16 / 2 and 32 / 8 heads of 128, vocabularies
151936 tied / 128256 untied, RoPE theta 1e6 / 5e5, RMSNorm eps 1e-6 / 1e-5,
LoRA r = 16), cut to two decoder layers so that the fp64 oracle can run every
step, batch 1 x 512 tokens:

* per-step loss against the oracle within 1e-3 relative (two steps, so the
  second loss also checks the optimizer step);
* the first step's LoRA gradients against the oracle's, at the whole-model
  tolerance of tests/test_gpu_model.py;
* the 3B shape cut to four layers, streamed through two slots, equals the
  resident run bit for bit (loss curve, gradients, logits).

This path runs everything the full configurations run at these widths: the
tcgen05 attention at GQA groups of 8 and 4, the 256-wide k / v projections
of the 3B shape, the tied 151936-row head.
"""
import dataclasses

import pytest
import torch

import synthetic as S
from oracle import train as OT
from test_gpu_model import _check_losses, _run, model_tolerance
from tolerances import check_model_grads

pytestmark = pytest.mark.gpu


def _cut(shape, n_layers):
    return dataclasses.replace(shape, name=f"{shape.name}-{n_layers}l", n_layers=n_layers)


@pytest.mark.parametrize("base", [S.QWEN3B, S.LLAMA8B])
def test_truncated_full_width_matches_oracle(lsq, base):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    shape, B, Sq, steps = _cut(base, 2), 1, 512, 2
    tr = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="host")
    losses, g0, _ = _run(tr, shape, B, Sq, steps)
    tr.close()
    layers = [S.layer_weights(shape, l) for l in range(shape.n_layers)]
    lora = [{n: {ab: t[ab] for ab in ("A", "B")} for n, t in per.items()} for per in S.lora_init(shape)]
    ids = [S.tokens(shape, B, Sq, step=t) for t in range(steps)]
    ol, og, _ = OT.train(shape, layers, S.embeddings(shape), lora, ids)
    _check_losses(losses, ol, shape.name)
    check_model_grads(tr.lora, g0, og, shape, model_tolerance(shape, B, Sq, og), what=shape.name)


def test_truncated_3b_streamed_equals_resident_bitwise(lsq):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    shape, B, Sq, steps = _cut(S.QWEN3B, 4), 1, 512, 3
    ref = StreamedLoraTrainer(shape, B, Sq, n_slots=None, init="device")
    rl, rg, rlog = _run(ref, shape, B, Sq, steps)
    ref.close()
    tr = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device")
    sl, sg, slog = _run(tr, shape, B, Sq, steps)
    uploads, _, _ = tr.stats()
    tr.close()
    assert uploads > shape.n_layers
    assert sl == rl
    assert torch.equal(sg, rg)
    assert torch.equal(slog, rlog)
