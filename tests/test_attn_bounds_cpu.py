"""The attention tolerance (attn_bounds.py) against a CPU model of the kernels'
arithmetic: fp32 products and sums with bf16 roundings exactly where the CUDA
kernels round (the probabilities entering P.V and P^T.dO, dS, the outputs; D
from the bf16 output).  The model's errors must sit inside the bound, and
plausible mistakes (D of the wrong row, dV from one head of a GQA group, a
transposed mask) must fall far outside it."""
import math

import torch

from attn_bounds import attention_bounds


def _bf(t):
    return t.to(torch.bfloat16).to(torch.float32)


def _model(q, k, v, do, shift_d=False, one_head_dv=False, mask_diag_off=False):
    B, S, Hq, hd = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    kk, vv = k.repeat_interleave(g, 2), v.repeat_interleave(g, 2)
    tau = 1.0 / math.sqrt(hd)
    mask = torch.triu(torch.ones(S, S, dtype=torch.bool), 0 if mask_diag_off else 1)
    mask[0, 0] = False
    s = (torch.einsum("bihd,bjhd->bhij", q, kk) * tau).masked_fill(mask, float("-inf"))
    m = s.max(-1, keepdim=True).values
    p = torch.exp(s - m)
    l = p.sum(-1, keepdim=True)
    o = _bf(torch.einsum("bhij,bjhd->bihd", _bf(p), vv) / l.squeeze(-1).permute(0, 2, 1)[..., None])
    P = torch.exp(s - (m + torch.log(l)))
    D = (do * o).sum(-1).permute(0, 2, 1)
    if shift_d:
        D = torch.roll(D, 1, dims=-1)
    dP = torch.einsum("bihd,bjhd->bhij", do, vv)
    dS = _bf(P * (dP - D[..., None]))
    dq = _bf(tau * torch.einsum("bhij,bjhd->bihd", dS, kk))
    dk = _bf((tau * torch.einsum("bhij,bihd->bjhd", dS, q)).reshape(B, S, Hkv, g, hd).sum(3))
    pdo = torch.einsum("bhij,bihd->bjhd", _bf(P), do).reshape(B, S, Hkv, g, hd)
    dv = _bf(pdo[:, :, :, 0] * g if one_head_dv else pdo.sum(3))
    return {"o": o, "dq": dq, "dk": dk, "dv": dv}


def _inputs(B=1, S=192, Hq=4, Hkv=2, hd=128, seed=0):
    g = torch.Generator().manual_seed(seed)
    return [_bf(torch.randn(B, S, h, hd, generator=g)) for h in (Hq, Hkv, Hkv, Hq)]


def _worst(got, bnd, name):
    return float(((got[name].double() - bnd[name]).abs() / bnd["b_" + name]).max())


def test_kernel_arithmetic_within_bound():
    for seed, shape in ((0, dict()), (1, dict(S=64, Hq=8, Hkv=1)), (2, dict(S=1))):
        q, k, v, do = _inputs(seed=seed, **shape)
        bnd = attention_bounds(q, k, v, do)
        got = _model(q, k, v, do)
        for name in ("o", "dq", "dk", "dv"):
            assert _worst(got, bnd, name) <= 1.0, (seed, name, _worst(got, bnd, name))
            if bnd[name].norm() > 0:
                rf = float((got[name].double() - bnd[name]).norm() / bnd[name].norm())
                assert rf <= 5e-3, (seed, name, rf)


def test_planted_mistakes_fall_outside_bound():
    q, k, v, do = _inputs(seed=3)
    bnd = attention_bounds(q, k, v, do)
    assert _worst(_model(q, k, v, do, shift_d=True), bnd, "dq") > 10
    assert _worst(_model(q, k, v, do, one_head_dv=True), bnd, "dv") > 10
    assert _worst(_model(q, k, v, do, mask_diag_off=True), bnd, "o") > 10
