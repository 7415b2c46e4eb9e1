"""Where the CUDA path stores values in bf16: a CPU model for the whole-model
gradient tolerance (test infrastructure).

The training step keeps every activation and every activation gradient in
bf16 between kernels (as the pages' bf16 trainer does): the layer input, the
normalised input, q / k (rotated by RoPE in their GEMM's epilogue) and v, the
attention output, the
residual stream after each fused o / down GEMM, the SwiGLU operands and
product, the final norm's output, and on the way back the logits' gradient
and the gradient of each of those.  This module re-runs the oracle's forward
and backward (oracle.decoder, fp64) with a bf16 rounding at exactly those
points: forward values are rounded, and the gradient that flows back through
each point is rounded too (a custom autograd function).  Nothing else is
rounded: the products inside a kernel stay fp64 here.

The LoRA gradients are sensitive to that storage rounding: at the test
shapes this model differs from the fp64 oracle by about 0.5% to 3% relative
Frobenius error per tensor, and the GPU's own difference from the oracle is
0.8 to 1.3 times this model's, tensor by tensor.  The whole-model tests
therefore hold each LoRA gradient tensor to twice this model's error against
the oracle (never tighter than the 5e-3 of a single GEMM): a kernel mistake
(a dropped term, a wrong index or sign) moves a gradient by far more than
its bf16 storage does.
"""
from __future__ import annotations

import torch

from oracle import decoder as D

F64 = torch.float64


def _bf16(x: torch.Tensor) -> torch.Tensor:
    return x.to(torch.float32).to(torch.bfloat16).to(F64)


ROUNDING = [True]   # False: the same graph without any rounding (equals the oracle; a CPU test checks it)


class _Stored(torch.autograd.Function):
    """A value stored in bf16 between kernels: the forward value is rounded
    (unless fwd is False, as for the fp32 logits) and so is its gradient
    (unless bwd is False)."""

    @staticmethod
    def forward(ctx, x, fwd, bwd):
        ctx.bwd = bwd
        return _bf16(x) if fwd and ROUNDING[0] else x.clone()

    @staticmethod
    def backward(ctx, g):
        return (_bf16(g) if ctx.bwd and ROUNDING[0] else g), None, None


def _st(x, fwd=True, bwd=True):
    return _Stored.apply(x, fwd, bwd)


def _layer(h, W, lora, shape, s):
    B, S, d = h.shape
    hd, nq, nkv = shape.hd, shape.n_q, shape.n_kv

    def lin(x, name):
        return D.lora_linear(x, W[name], lora[name]["A"], lora[name]["B"], s)

    x = _st(D.rmsnorm(h, W["ln1"], shape.eps))
    v = _st(lin(x, "v")).reshape(B, S, nkv, hd)
    if hd in (64, 128, 256):
        # RoPE in the q / k GEMM epilogue: one rounding after the rotation; on the way back the
        # tcgen05 attention (hd 128, up to 512 positions) rotates the fp32 gradient before its one
        # rounding, the other attention kernels round it, then a RoPE pass rounds it again
        fused_bwd = hd == 128 and S <= 512
        q = _st(D.rope(_st(lin(x, "q"), fwd=False).reshape(B, S, nq, hd), shape.theta), bwd=not fused_bwd)
        k = _st(D.rope(_st(lin(x, "k"), fwd=False).reshape(B, S, nkv, hd), shape.theta), bwd=not fused_bwd)
    else:
        q = _st(D.rope(_st(lin(x, "q")).reshape(B, S, nq, hd), shape.theta))
        k = _st(D.rope(_st(lin(x, "k")).reshape(B, S, nkv, hd), shape.theta))
    a = _st(D.causal_gqa_attention(q, k, v)).reshape(B, S, d)
    h = _st(h + lin(a, "o"))                      # the residual add is fused into the o GEMM
    x = _st(D.rmsnorm(h, W["ln2"], shape.eps))
    m = _st(D.silu(_st(lin(x, "gate"))) * _st(lin(x, "up")))
    return _st(h + lin(m, "down"))                # and into the down GEMM


def _logits(ids, layers, emb, lora, shape, s):
    h = emb["embed"][ids.long()]
    for l, W in enumerate(layers):
        h = _layer(h, W, lora[l], shape, s)
    hn = _st(D.rmsnorm(h, emb["final_norm"], shape.eps))
    return _st(hn @ emb["lm_head"].T, fwd=False)  # fp32 logits, bf16 gradient


def _leaves(lora):
    return [{n: {ab: t[ab].detach().clone().requires_grad_(True) for ab in ("A", "B")} for n, t in per.items()}
            for per in lora]


def _grads(loss, leaves):
    flat = [leaves[l][n][ab] for l in range(len(leaves)) for n in leaves[l] for ab in ("A", "B")]
    gr = iter(torch.autograd.grad(loss, flat))
    return [{n: {"A": next(gr), "B": next(gr)} for n in per} for per in leaves]


def sft_grads(ids, layers, emb, lora, shape):
    """LoRA gradients of the causal-LM loss with bf16 storage; layers / emb /
    lora as oracle.decoder.model_loss_and_grads takes them (fp64)."""
    leaves = _leaves(lora)
    loss = D.cross_entropy_next_token(_logits(ids, layers, emb, leaves, shape, shape.s), ids)
    return _grads(loss, leaves)


def dpo_grads(ids, layers, emb, lora, shape, beta):
    """LoRA gradients of the DPO loss with bf16 storage (the reference, the
    base with the adapters off, needs no gradient)."""
    leaves = _leaves(lora)
    with torch.no_grad():
        ref = D.sequence_logprob(_logits(ids, layers, emb, lora, shape, 0.0), ids)
    pi = D.sequence_logprob(_logits(ids, layers, emb, leaves, shape, shape.s), ids)
    return _grads(D.dpo_loss(pi, ref, beta), leaves)


def tolerance(ref_grads, model_grads, floor=5e-3, factor=2.0):
    """(layer, name, "A"|"B") -> factor x this model's relative Frobenius error
    against the oracle's gradient, at least floor."""
    def rf(a, b):
        return float(torch.linalg.norm(a - b) / torch.linalg.norm(b))
    tol = {}
    for l, per in enumerate(ref_grads):
        for n, t in per.items():
            for ab in ("A", "B"):
                tol[(l, n, ab)] = max(floor, factor * rf(model_grads[l][n][ab], t[ab]))
    return tol
