"""Frozen-base NF4 linear with a LoRA adapter, forward and backward, in fp64 (oracle).

TEST INFRASTRUCTURE ONLY: see ``oracle/__init__.py``.

The pages describe the trainer as LoRA on a frozen NF4 base in which the
adapter is the only trained and permanently resident part (themenonlab blog,
"The trick: layer streaming"; soup-cli 0.72.0 -> 0.72.2 diff, docs "Layer
Streaming", config keys lora.r / lora.alpha), and they test that the first
layer still receives gradients (CHANGELOG [0.72.2], "Correctness").  The maths is the plain LoRA
definition (Hu et al. 2021): with W' = deq(W) [N, K], A [r, K], B [N, r] and
s = alpha / r,

    Y  = X W'^T + s (X A^T) B^T
    U  = X A^T                      (kept for the backward)
    G  = dY B
    dX = dY W' + s G A
    dB = s dY^T U
    dA = s G^T X

There is no gradient for the frozen W'.  Every operand is taken as given
(bf16 values widened to fp64); nothing is rounded inside.
"""
from __future__ import annotations

import numpy as np


def lora_forward(X, Wd, A, B, s):
    """-> (Y [M,N], U [M,r]) in fp64."""
    X, Wd, A, B = (np.asarray(t, dtype=np.float64) for t in (X, Wd, A, B))
    U = X @ A.T
    Y = X @ Wd.T + s * (U @ B.T)
    return Y, U


def lora_backward(X, Wd, A, B, s, dY):
    """-> (dX [M,K], dA [r,K], dB [N,r], G [M,r]) in fp64."""
    X, Wd, A, B, dY = (np.asarray(t, dtype=np.float64) for t in (X, Wd, A, B, dY))
    U = X @ A.T
    G = dY @ B
    dX = dY @ Wd + s * (G @ A)
    dB = s * (dY.T @ U)
    dA = s * (G.T @ X)
    return dX, dA, dB, G


def lora_loss(X, Wd, A, B, s, dY):
    """<dY, Y>: the scalar whose gradients are the ones lora_backward returns."""
    Y, _ = lora_forward(X, Wd, A, B, s)
    return float(np.sum(np.asarray(dY, dtype=np.float64) * Y))
