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


LOG2E = 1.4426950408889634


def _online_o(s, vv, chunk=64, thresh=8.0):
    """The forward's online softmax: 64-key chunks, a running max in log2 units that is kept
    while a chunk's max exceeds it by at most 8 (else O and l are rescaled), bf16 P into P.V."""
    s2 = s * LOG2E
    B, H, S, _ = s.shape
    m = torch.full((B, H, S), float("-inf"))
    l = torch.zeros(B, H, S)
    O = torch.zeros(B, H, S, vv.shape[-1])
    for j0 in range(0, S, chunk):
        sc = s2[..., j0:j0 + chunk]
        mc = sc.max(-1).values
        need = mc > m + thresh
        alpha = torch.where(need, torch.exp2(m - mc), torch.ones_like(m))
        O, l = O * alpha[..., None], l * alpha
        m = torch.where(need, mc, m)
        p = torch.exp2(sc - m[..., None])
        l = l + p.sum(-1)
        O = O + torch.einsum("bhij,bjhd->bhid", _bf(p), vv[:, j0:j0 + chunk])
    return _bf((O / l[..., None]).permute(0, 2, 1, 3)), m, l


def _model(q, k, v, do, shift_d=False, one_head_dv=False, mask_diag_off=False, online=False):
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
    if online:
        o = _online_o(s, vv)[0]
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


def _ramped(q, k, v, do):
    """Keys whose scores grow along the sequence (key j scaled by 1 + 8 j / S): each chunk's max
    jumps past the running one, so the online forward rescales O again and again."""
    S = k.shape[1]
    ramp = _bf(k * (1.0 + 8.0 * torch.arange(S, dtype=torch.float32) / S)[None, :, None, None])
    return q, ramp, v, do


def test_online_softmax_rescales_on_ramped_keys():
    q, k, v, do = _ramped(*_inputs(seed=4, S=256))
    s = torch.einsum("bihd,bjhd->bhij", q, k.repeat_interleave(2, 2)) / math.sqrt(128)
    s = s.masked_fill(torch.triu(torch.ones(256, 256, dtype=torch.bool), 1), float("-inf"))
    _, m, l = _online_o(s, v.repeat_interleave(2, 2))
    # the kept max is within 8 (log2 units) of the true one, and lse is exact whichever was kept
    true = s.max(-1).values * LOG2E
    assert bool(((true - m) <= 8.0 + 1e-4).all()) and bool((m <= true + 1e-4).all())
    lse = (m + torch.log2(l)) / LOG2E
    assert torch.allclose(lse, torch.logsumexp(s, -1), atol=1e-4)
    # rescales happened: some rows' kept max moved in a later chunk
    first = s[..., :64].max(-1).values * LOG2E
    assert bool((m > first + 8.0).any())


def test_kernel_arithmetic_within_bound():
    cases = [(0, dict(), False, False), (1, dict(S=64, Hq=8, Hkv=1), False, False), (2, dict(S=1), False, False),
             (0, dict(), True, False), (5, dict(S=512, Hq=2, Hkv=1), True, False), (6, dict(S=256), True, True)]
    for seed, shape, online, ramped in cases:
        q, k, v, do = _inputs(seed=seed, **shape)
        if ramped:
            q, k, v, do = _ramped(q, k, v, do)
        bnd = attention_bounds(q, k, v, do)
        got = _model(q, k, v, do, online=online)
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
    assert _worst(_model(q, k, v, do, mask_diag_off=True, online=True), bnd, "o") > 10
