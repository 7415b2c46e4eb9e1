"""Whole-model LoRA training steps on the NF4 base, in fp64 (oracle).

TEST INFRASTRUCTURE ONLY: see ``oracle/__init__.py``.

One step, as the pages' trainer runs it (soup-cli 0.72.0 -> 0.72.2 diff,
CHANGELOG [0.72.2]: batch of token ids, causal-LM SFT loss, gradients to the
LoRA adapters only, optimizer step):

1. the frozen linears are the oracle's own NF4 quantisation of the bf16 base,
   dequantised (``oracle.nf4``); embeddings, lm_head and RMSNorm gains stay bf16;
2. the LoRA operands are the fp32 masters rounded to bf16 (the trainer keeps
   fp32 masters and computes with bf16 copies);
3. loss and LoRA gradients in fp64 (``oracle.decoder``);
4. AdamW on the masters.
"""
from __future__ import annotations

from typing import Dict, List

import numpy as np
import torch

from . import nf4
from .decoder import DPO_BETA, F64, adamw, model_dpo_loss_and_grads, model_loss_and_grads


def dequantized_layer(Wbf16: Dict[str, torch.Tensor], double_quant: bool = False) -> Dict[str, torch.Tensor]:
    """fp64 weights the layer computes with: NF4 quantise, then dequantise; with
    double_quant the absmax array goes through its 8-bit second level first."""
    out = {}
    for name, w in Wbf16.items():
        if name in ("ln1", "ln2"):
            out[name] = w.to(F64)
            continue
        a = w.float().numpy()
        N, K = a.shape
        packed, am = nf4.quantize(a)
        if double_quant:
            am = nf4.double_quantized(am)
        out[name] = torch.from_numpy(nf4.dequantize_f64(packed, am, N, K))
    return out


def operand(master: torch.Tensor) -> torch.Tensor:
    """bf16 operand copy of an fp32 master, widened to fp64."""
    return torch.from_numpy(nf4.bf16_round(master.detach().to(torch.float32).numpy()).astype(np.float64))


def train(shape, layers_bf16, emb_bf16, lora_masters, ids_per_step: List[torch.Tensor],
          lr: float = 2e-5, double_quant: bool = False):
    """Run len(ids_per_step) steps; returns (losses, grads of the first step, final masters)."""
    layers = [dequantized_layer(W, double_quant) for W in layers_bf16]
    emb = {k: v.to(F64) for k, v in emb_bf16.items()}
    masters = [{n: {ab: t[ab].detach().to(F64).clone() for ab in ("A", "B")} for n, t in per.items()}
               for per in lora_masters]
    mom = [{n: {ab: torch.zeros_like(t[ab]) for ab in ("A", "B")} for n, t in per.items()} for per in masters]
    vel = [{n: {ab: torch.zeros_like(t[ab]) for ab in ("A", "B")} for n, t in per.items()} for per in masters]
    losses, first_grads = [], None
    for step, ids in enumerate(ids_per_step, start=1):
        ops = [{n: {ab: operand(t[ab]) for ab in ("A", "B")} for n, t in per.items()} for per in masters]
        loss, grads = model_loss_and_grads(ids, layers, emb, ops, shape)
        losses.append(loss)
        if first_grads is None:
            first_grads = grads
        for l, per in enumerate(masters):
            for n in per:
                for ab in ("A", "B"):
                    # the master is an fp32 tensor in the trainer: keep it rounded to fp32
                    p, m, v = adamw(per[n][ab], grads[l][n][ab], mom[l][n][ab], vel[l][n][ab], step, lr=lr)
                    per[n][ab] = p.to(torch.float32).to(F64)
                    mom[l][n][ab], vel[l][n][ab] = m, v
    return losses, first_grads, masters


def dpo_step(shape, layers_bf16, emb_bf16, lora_masters, ids: torch.Tensor, beta: float = DPO_BETA):
    """One DPO forward/backward on the NF4 base (reference = the same base with
    the adapters off): -> (loss, grads, policy sequence log-probs, reference ones)."""
    layers = [dequantized_layer(W) for W in layers_bf16]
    emb = {k: v.to(F64) for k, v in emb_bf16.items()}
    ops = [{n: {ab: operand(t[ab]) for ab in ("A", "B")} for n, t in per.items()} for per in lora_masters]
    return model_dpo_loss_and_grads(ids, layers, emb, ops, shape, beta)
