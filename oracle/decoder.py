"""Llama/Qwen decoder stack around the NF4-LoRA linears, in fp64 (oracle).

TEST INFRASTRUCTURE ONLY: see ``oracle/__init__.py``.

The pages restrict streaming to Llama and Qwen models (soup-cli 0.72.0 ->
0.72.2 diff, docs "Layer Streaming", "Honest scope"), name the task (causal-LM
SFT, ``task: sft``), say the streamer applies gradient checkpointing layer by
layer (same section, example config) and keep the embedding and lm_head on the
GPU in full precision (same section, "NF4 streaming").  They give no
formula.  The forward here is the plain definition of a pre-norm Llama/Qwen
decoder layer, written in PyTorch CPU ops in float64:

    x  = RMSNorm(h) * g1                        RMSNorm(x) = x / sqrt(mean(x^2) + eps)
    q, k, v = LoRA-linears of x                 (heads of size hd = d / n_q)
    q, k = RoPE(q), RoPE(k)                     rotate-half, inv_freq_i = theta^(-2i/hd)
    a  = softmax(q k^T / sqrt(hd) + causal) v   GQA: query head j uses kv head j // (n_q / n_kv)
    h  = h + o(a)
    x  = RMSNorm(h) * g2
    h  = h + down(silu(gate(x)) * up(x))

Readings where the pages are silent: no biases (the workloads give shapes only);
no RoPE frequency scaling; loss = mean next-token NLL over B*(S-1) positions.
The backward is the exact gradient of this forward, taken by torch.autograd in
float64 (a library primitive); its correctness is pinned by central finite
differences in the tests.  Checkpointing changes no value, so the oracle is
resident and computes each layer once.
"""
from __future__ import annotations

import math
from typing import Dict, List

import torch

F64 = torch.float64


def rmsnorm(x: torch.Tensor, g: torch.Tensor, eps: float) -> torch.Tensor:
    return x / torch.sqrt((x * x).mean(dim=-1, keepdim=True) + eps) * g


def rope_tables(S: int, hd: int, theta: float):
    i = torch.arange(hd // 2, dtype=F64)
    inv_freq = theta ** (-2.0 * i / hd)
    ang = torch.arange(S, dtype=F64)[:, None] * inv_freq[None, :]
    return torch.cos(ang), torch.sin(ang)


def rope(x: torch.Tensor, theta: float) -> torch.Tensor:
    """x [B, S, H, hd] -> rotate-half RoPE at positions 0..S-1."""
    B, S, H, hd = x.shape
    cos, sin = rope_tables(S, hd, theta)
    cos = cos[None, :, None, :]
    sin = sin[None, :, None, :]
    x1, x2 = x[..., : hd // 2], x[..., hd // 2:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def causal_gqa_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
    """q [B,S,Hq,hd], k/v [B,S,Hkv,hd] -> [B,S,Hq,hd]; softmax in fp64."""
    B, S, Hq, hd = q.shape
    Hkv = k.shape[2]
    group = Hq // Hkv
    kk = k.repeat_interleave(group, dim=2)
    vv = v.repeat_interleave(group, dim=2)
    scores = torch.einsum("bihd,bjhd->bhij", q, kk) / math.sqrt(hd)
    mask = torch.triu(torch.ones(S, S, dtype=torch.bool), diagonal=1)
    scores = scores.masked_fill(mask, float("-inf"))
    p = torch.softmax(scores, dim=-1)
    return torch.einsum("bhij,bjhd->bihd", p, vv)


def silu(x: torch.Tensor) -> torch.Tensor:
    return x / (1.0 + torch.exp(-x))


def lora_linear(x: torch.Tensor, Wd: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float) -> torch.Tensor:
    """y = x W'^T + s (x A^T) B^T."""
    return x @ Wd.T + s * ((x @ A.T) @ B.T)


def decoder_layer(h: torch.Tensor, W: Dict[str, torch.Tensor], lora: Dict[str, Dict[str, torch.Tensor]],
                  shape, s: float) -> torch.Tensor:
    """h [B, S, d] fp64 -> next residual stream [B, S, d]."""
    B, S, d = h.shape
    hd, nq, nkv = shape.hd, shape.n_q, shape.n_kv

    def lin(x, name):
        return lora_linear(x, W[name], lora[name]["A"], lora[name]["B"], s)

    x = rmsnorm(h, W["ln1"], shape.eps)
    q = lin(x, "q").reshape(B, S, nq, hd)
    k = lin(x, "k").reshape(B, S, nkv, hd)
    v = lin(x, "v").reshape(B, S, nkv, hd)
    q = rope(q, shape.theta)
    k = rope(k, shape.theta)
    a = causal_gqa_attention(q, k, v).reshape(B, S, d)
    h = h + lin(a, "o")
    x = rmsnorm(h, W["ln2"], shape.eps)
    m = silu(lin(x, "gate")) * lin(x, "up")
    return h + lin(m, "down")


def cross_entropy_next_token(logits: torch.Tensor, ids: torch.Tensor) -> torch.Tensor:
    """mean NLL of ids[:, 1:] under logits[:, :-1]; logits [B,S,V] fp64."""
    lg = logits[:, :-1, :]
    tgt = ids[:, 1:].long()
    lse = torch.logsumexp(lg, dim=-1)
    picked = torch.gather(lg, -1, tgt[..., None])[..., 0]
    return (lse - picked).mean()


def model_loss(ids: torch.Tensor, layers: List[Dict[str, torch.Tensor]], emb: Dict[str, torch.Tensor],
               lora: List[Dict[str, Dict[str, torch.Tensor]]], shape) -> torch.Tensor:
    """Causal-LM loss of the whole stack.  All tensors fp64; ids int [B, S]."""
    h = emb["embed"][ids.long()]
    s = shape.s
    for l, W in enumerate(layers):
        h = decoder_layer(h, W, lora[l], shape, s)
    h = rmsnorm(h, emb["final_norm"], shape.eps)
    logits = h @ emb["lm_head"].T
    return cross_entropy_next_token(logits, ids)


def model_loss_and_grads(ids, layers, emb, lora, shape):
    """-> (loss, grads) with grads[l][name]["A"|"B"] = d loss / d LoRA operand."""
    leaves = [{n: {"A": t["A"].detach().clone().requires_grad_(True),
                   "B": t["B"].detach().clone().requires_grad_(True)} for n, t in per.items()}
              for per in lora]
    loss = model_loss(ids, layers, emb, leaves, shape)
    flat = [leaves[l][n][ab] for l in range(len(leaves)) for n in leaves[l] for ab in ("A", "B")]
    gr = torch.autograd.grad(loss, flat)
    grads, it = [], iter(gr)
    for per in leaves:
        grads.append({n: {"A": next(it), "B": next(it)} for n in per})
    return float(loss.detach()), grads


# ---------------------------------------------------------------- preference loss (DPO)
# The pages name DPO among the preference losses that streaming serves and say
# the reference model is the same streamed base with the adapters switched off
# (aiany.app listing, "How It Works (concise)"; soup-cli docs "Layer
# Streaming", preference losses v0.72.4).  They give no formula; the reading is
# the DPO objective of Rafailov et al. (2023, eq. 7):
#   z_i  = beta * ((pi(y_c) - ref(y_c)) - (pi(y_r) - ref(y_r)))
#   loss = mean_i -log sigmoid(z_i)
# over pairs i of sequences (chosen = row 2i, rejected = row 2i+1), where pi(y)
# and ref(y) are the summed next-token log-probabilities of a whole sequence
# (synthetic ids have no prompt/response split, so every position t < S-1
# counts) under the adapted model and under the same base with the LoRA path
# off (s = 0).  beta = 0.1 (reading).

DPO_BETA = 0.1


def sequence_logprob(logits: torch.Tensor, ids: torch.Tensor) -> torch.Tensor:
    """Summed log p(ids[b, t+1] | logits[b, t]) over t < S-1, per sequence -> [B] (fp64)."""
    lg = logits[:, :-1, :]
    tgt = ids[:, 1:].long()
    logp = lg - torch.logsumexp(lg, dim=-1, keepdim=True)
    return torch.gather(logp, -1, tgt[..., None])[..., 0].sum(dim=1)


def dpo_loss(pi_logp: torch.Tensor, ref_logp: torch.Tensor, beta: float = DPO_BETA) -> torch.Tensor:
    """DPO loss over pairs (rows 2i, 2i+1) = (chosen, rejected) of [2P] sequence log-probs."""
    pc, pr = pi_logp[0::2], pi_logp[1::2]
    rc, rr = ref_logp[0::2], ref_logp[1::2]
    z = beta * ((pc - rc) - (pr - rr))
    return torch.nn.functional.softplus(-z).mean()  # -log sigmoid(z) = log(1 + exp(-z))


def model_logits(ids, layers, emb, lora, shape, s: float) -> torch.Tensor:
    """Logits [B, S, V] of the stack with LoRA scale s (s = 0: the base alone)."""
    h = emb["embed"][ids.long()]
    for l, W in enumerate(layers):
        h = decoder_layer(h, W, lora[l], shape, s)
    h = rmsnorm(h, emb["final_norm"], shape.eps)
    return h @ emb["lm_head"].T


def model_dpo_loss_and_grads(ids, layers, emb, lora, shape, beta: float = DPO_BETA):
    """-> (loss, grads, policy_logp, ref_logp); grads[l][name]["A"|"B"] = d loss / d LoRA operand."""
    leaves = [{n: {"A": t["A"].detach().clone().requires_grad_(True),
                   "B": t["B"].detach().clone().requires_grad_(True)} for n, t in per.items()}
              for per in lora]
    with torch.no_grad():
        ref = sequence_logprob(model_logits(ids, layers, emb, lora, shape, 0.0), ids)
    pi = sequence_logprob(model_logits(ids, layers, emb, leaves, shape, shape.s), ids)
    loss = dpo_loss(pi, ref, beta)
    flat = [leaves[l][n][ab] for l in range(len(leaves)) for n in leaves[l] for ab in ("A", "B")]
    gr = torch.autograd.grad(loss, flat)
    grads, it = [], iter(gr)
    for per in leaves:
        grads.append({n: {"A": next(it), "B": next(it)} for n in per})
    return float(loss.detach()), grads, pi.detach(), ref


def adamw(master, grad, m, v, t: int, lr: float = 2e-5, b1: float = 0.9, b2: float = 0.999,
          eps: float = 1e-8, wd: float = 0.0):
    """One AdamW step in fp64 (Loshchilov & Hutter); returns (master, m, v).

    The pages' optimizer is PagedAdamW8bit (CHANGELOG [0.72.2], "Measured on a
    4 GB RTX 3050 Laptop"); the reading here is plain AdamW with the pages'
    lr 2e-5 and the usual betas, fp32 master weights.
    """
    master = torch.as_tensor(master, dtype=F64)
    grad = torch.as_tensor(grad, dtype=F64)
    m = b1 * torch.as_tensor(m, dtype=F64) + (1 - b1) * grad
    v = b2 * torch.as_tensor(v, dtype=F64) + (1 - b2) * grad * grad
    mhat = m / (1 - b1 ** t)
    vhat = v / (1 - b2 ** t)
    master = master - lr * (mhat / (torch.sqrt(vhat) + eps) + wd * master)
    return master, m, v
