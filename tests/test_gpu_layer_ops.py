"""GPU parity of the decoder-layer kernels against the fp64 oracle (forward
values, and backward values against torch.autograd through the oracle's
forward in float64)."""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import decoder as D
from attn_bounds import attention_bounds
from attn_model import frobenius_tolerance
from tolerances import assert_close, assert_close_ew, assert_within_bound

pytestmark = pytest.mark.gpu
F64 = torch.float64


def _rand(shape, std=1.0, stream=0):
    return S.bf16(S.normal_f32(S.DATA_SEED, 9000 + stream, shape, std))


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _grad(fn, inputs, dy):
    xs = [x.detach().to(F64).requires_grad_(True) for x in inputs]
    out = fn(*xs)
    gr = torch.autograd.grad(out, xs, grad_outputs=dy.to(F64))
    return out.detach(), gr


@pytest.mark.parametrize("M,d,eps", [(130, 576, 1e-5), (64, 4096, 1e-5), (1, 256, 1e-5), (512, 2048, 1e-6),
                                     (8, 5120, 1e-5), (3, 9216, 1e-5)])
def test_rmsnorm_fwd_bwd(lsq, M, d, eps):
    x = _rand((M, d), 2.0, 1)
    g = _rand((d,), 0.3, 2) + 1
    g = g.to(torch.bfloat16)
    dy = _rand((M, d), 1.0, 3)
    res = _rand((M, d), 1.0, 4)
    y = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    rstd = torch.empty(M, dtype=torch.float32, device="cuda")
    lsq.lsq_rmsnorm_fwd(x.cuda(), g.cuda(), y, rstd, M, d, eps)
    out = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    lsq.lsq_rmsnorm_bwd(dy.cuda(), x.cuda(), g.cuda(), rstd, res.cuda(), out, M, d)
    torch.cuda.synchronize()
    ref, (dx, _) = _grad(lambda a, b: D.rmsnorm(a, b, eps), [x, g], dy)
    assert_close_ew(_np(y), ref.numpy(), what="rmsnorm y")
    rr = 1.0 / np.sqrt((_np(x) ** 2).mean(-1) + eps)
    assert_close(rstd.cpu().numpy(), rr, rel=1e-6, max_rms=1e-5, what="rstd")
    assert_close_ew(_np(out), dx.numpy() + _np(res), what="rmsnorm dx + res")
    out0 = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")   # no residual gradient to add
    lsq.lsq_rmsnorm_bwd(dy.cuda(), x.cuda(), g.cuda(), rstd, None, out0, M, d)
    torch.cuda.synchronize()
    assert_close_ew(_np(out0), dx.numpy(), what="rmsnorm dx")


@pytest.mark.parametrize("B,Sq,H,hd,theta", [(2, 300, 4, 64, 1e4), (1, 512, 8, 128, 5e5), (1, 50, 3, 24, 1e4),
                                             (1, 512, 16, 128, 1e6)])
def test_rope_fwd_and_transpose(lsq, B, Sq, H, hd, theta):
    x = _rand((B, Sq, H, hd), 1.0, 5)
    dy = _rand((B, Sq, H, hd), 1.0, 6)
    xg = x.cuda().contiguous()
    lsq.lsq_rope(xg, B, Sq, H, hd, theta, 0)
    dg = dy.cuda().contiguous()
    lsq.lsq_rope(dg, B, Sq, H, hd, theta, 1)
    torch.cuda.synchronize()
    ref, (dx,) = _grad(lambda a: D.rope(a, theta), [x], dy)
    assert_close_ew(_np(xg), ref.numpy(), what="rope")
    assert_close_ew(_np(dg), dx.numpy(), what="rope transpose")


def test_swiglu_fwd_bwd(lsq):
    n = 4096 * 3
    g, u, dm = _rand((n,), 2.0, 7), _rand((n,), 1.0, 8), _rand((n,), 1.0, 9)
    m = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    lsq.lsq_swiglu_fwd(g.cuda(), u.cuda(), m, n)
    gg, uu = g.cuda().clone(), u.cuda().clone()
    lsq.lsq_swiglu_bwd(dm.cuda(), gg, uu, gg, uu, n)   # in place
    torch.cuda.synchronize()
    ref, (dg, du) = _grad(lambda a, b: D.silu(a) * b, [g, u], dm)
    assert_close_ew(_np(m), ref.numpy(), what="swiglu")
    assert_close_ew(_np(gg), dg.numpy(), what="dg")
    assert_close_ew(_np(uu), du.numpy(), what="du")


def _attn_case(B, Sq, Hq, Hkv, hd, seed):
    q = _rand((B, Sq, Hq, hd), 1.0, 20 + seed)
    k = _rand((B, Sq, Hkv, hd), 1.0, 21 + seed)
    v = _rand((B, Sq, Hkv, hd), 1.0, 22 + seed)
    do = _rand((B, Sq, Hq, hd), 1.0, 23 + seed)
    return q, k, v, do


@pytest.mark.parametrize("B,Sq,Hq,Hkv,hd,ramp", [(1, 512, 9, 3, 64, False), (2, 200, 4, 1, 128, False),
                                                 (1, 64, 2, 2, 64, False), (1, 1, 4, 2, 128, False),
                                                 (2, 130, 8, 2, 128, False), (2, 512, 32, 8, 128, False),
                                                 (1, 384, 4, 4, 128, False), (1, 300, 7, 1, 128, False),
                                                 (2, 256, 6, 2, 128, False), (1, 512, 16, 2, 128, False),
                                                 (1, 512, 8, 2, 128, True), (2, 300, 4, 1, 128, True)])
def test_attention_fwd_bwd(lsq, B, Sq, Hq, Hkv, hd, ramp):
    """ramp: key j scaled by 1 + 8 j / S, so that each 64-key chunk's max jumps past the running
    one and the forward's online softmax rescales its accumulator again and again."""
    q, k, v, do = _attn_case(B, Sq, Hq, Hkv, hd, Sq)
    if ramp:
        k = (k.float() * (1.0 + 8.0 * torch.arange(Sq, dtype=torch.float32) / Sq)[None, :, None, None]).to(k.dtype)
    o = torch.empty(B, Sq, Hq, hd, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device="cuda")
    lsq.lsq_attention_fwd(q.cuda(), k.cuda(), v.cuda(), o, lse, B, Sq, Hq, Hkv, hd)
    dq = torch.empty_like(o)
    dk = torch.empty(B, Sq, Hkv, hd, dtype=torch.bfloat16, device="cuda")
    dv = torch.empty_like(dk)
    ws = torch.empty(lsq.lsq_attention_bwd_workspace_size(B, Sq, Hq), dtype=torch.uint8, device="cuda")
    lsq.lsq_attention_bwd(q.cuda(), k.cuda(), v.cuda(), o, lse, do.cuda(), dq, dk, dv, B, Sq, Hq, Hkv, hd, ws)
    torch.cuda.synchronize()
    ref, (rq, rk, rv) = _grad(D.causal_gqa_attention, [q, k, v], do)
    # lse of the scaled scores
    kk = k.to(F64).repeat_interleave(Hq // Hkv, dim=2)
    sc = torch.einsum("bihd,bjhd->bhij", q.to(F64), kk) / math.sqrt(hd)
    sc = sc.masked_fill(torch.triu(torch.ones(Sq, Sq, dtype=torch.bool), 1), float("-inf"))
    assert_close(lse.cpu().numpy(), torch.logsumexp(sc, -1).numpy(), rel=1e-5, max_rms=1e-4, what="lse")
    # Element by element within the first-order bound of the kernels' bf16
    # roundings (P and dS enter the tensor cores as bf16, D is formed from the
    # bf16 output; attn_bounds.py), plus relative Frobenius 5e-3.  The bound's
    # exact values are the oracle's (autograd through its forward).
    bnd = attention_bounds(q, k, v, do)
    for name, want in (("o", ref), ("dq", rq), ("dk", rk), ("dv", rv)):
        assert torch.allclose(bnd[name], want, rtol=1e-9, atol=1e-12), name
    # relative Frobenius: the GEMMs' 5e-3; with a sharp softmax (ramped keys) dS = P (dP - D) cancels
    # and the bf16 roundings alone move dq and dk by about that much, so there each output is held
    # to twice the CPU model of the kernels' roundings (attn_model.py), never below 5e-3
    tol = frobenius_tolerance(q, k, v, do, bnd) if ramp else {n: 5e-3 for n in ("o", "dq", "dk", "dv")}
    assert_within_bound(_np(o), ref.numpy(), bnd["b_o"].numpy(), rel=tol["o"], what="attn out")
    assert_within_bound(_np(dq), rq.numpy(), bnd["b_dq"].numpy(), rel=tol["dq"], what="dq")
    assert_within_bound(_np(dk), rk.numpy(), bnd["b_dk"].numpy(), rel=tol["dk"], what="dk")
    assert_within_bound(_np(dv), rv.numpy(), bnd["b_dv"].numpy(), rel=tol["dv"], what="dv")


def test_attention_deterministic(lsq):
    B, Sq, Hq, Hkv, hd = 2, 256, 8, 2, 128
    q, k, v, do = (t.cuda() for t in _attn_case(B, Sq, Hq, Hkv, hd, 7))
    outs = []
    for _ in range(2):
        o = torch.empty(B, Sq, Hq, hd, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device="cuda")
        lsq.lsq_attention_fwd(q, k, v, o, lse, B, Sq, Hq, Hkv, hd)
        dq, dk, dv = torch.empty_like(o), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(lsq.lsq_attention_bwd_workspace_size(B, Sq, Hq), dtype=torch.uint8, device="cuda")
        lsq.lsq_attention_bwd(q, k, v, o, lse, do, dq, dk, dv, B, Sq, Hq, Hkv, hd, ws)
        outs.append((o, lse, dq, dk, dv))
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


@pytest.mark.parametrize("B,Sq,V", [(2, 64, 1000), (1, 512, 49152), (1, 96, 128256), (2, 40, 1002)])
def test_cross_entropy(lsq, B, Sq, V):
    """Small, odd and 8B-sized vocabularies (128256) against the oracle's loss and gradient."""
    logits = torch.from_numpy(S.normal_f32(S.DATA_SEED, 77, (B * Sq, V), 2.0))
    ids = S.uniform_ids(S.DATA_SEED, 78, (B, Sq), V)
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    dl = torch.empty(B * Sq, V, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lsq.lsq_xent_workspace_size(B * Sq), dtype=torch.uint8, device="cuda")
    lsq.lsq_xent_fwd_bwd(logits.cuda(), ids.cuda(), B, Sq, V, loss, dl, ws)
    torch.cuda.synchronize()
    lg = logits.to(F64).reshape(B, Sq, V).requires_grad_(True)
    ref = D.cross_entropy_next_token(lg, ids)
    (g,) = torch.autograd.grad(ref, [lg])
    assert abs(loss.item() - ref.item()) <= 1e-5 * abs(ref.item())
    assert_close_ew(_np(dl), g.reshape(B * Sq, V).numpy(), what="dlogits")


def test_embed_gather_exact(lsq):
    V, d, M = 1000, 256, 300
    table = _rand((V, d), 1.0, 40)
    ids = S.uniform_ids(S.DATA_SEED, 41, (M,), V)
    h = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    lsq.lsq_embed_gather(ids.cuda(), table.cuda(), h, M, d, V)
    torch.cuda.synchronize()
    assert torch.equal(h.cpu(), table[ids.long()])


def test_adamw_matches_oracle(lsq):
    n = 10000
    p = torch.from_numpy(S.normal_f32(1, 50, (n,)))
    m = torch.zeros(n)
    v = torch.zeros(n)
    pg, mg, vg = p.cuda(), m.cuda(), v.cuda()
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    ref = (p.to(F64), m.to(F64), v.to(F64))
    for t in range(1, 4):
        g = torch.from_numpy(S.normal_f32(1, 50 + t, (n,), 1e-2))
        lsq.lsq_adamw_step(pg, g.cuda(), mg, vg, pb, n, t, 1e-3, 0.9, 0.999, 1e-8, 0.01)
        ref = D.adamw(ref[0], g, ref[1], ref[2], t, lr=1e-3, wd=0.01)
    torch.cuda.synchronize()
    assert_close(pg.cpu().numpy(), ref[0].numpy(), rel=1e-6, max_rms=1e-6, what="adamw p")
    assert torch.equal(pb.cpu(), pg.cpu().to(torch.bfloat16))


@pytest.mark.parametrize("B,Sq,Hq,Hkv,hd,theta", [(1, 384, 4, 4, 128, 5e5), (2, 130, 8, 2, 128, 1e4),
                                                  (1, 300, 7, 1, 128, 1e6), (1, 512, 9, 3, 64, 1e4)])
def test_attention_bwd_with_rope_transpose(lsq, B, Sq, Hq, Hkv, hd, theta):
    """lsq_attention_bwd_ex with a RoPE table returns the gradients of the
    unrotated q and k: the transpose of the rotation applied to the attention
    gradients (in fp32 before the one rounding on the tcgen05 path, in a pass
    over the bf16 gradients on the other), against the oracle's RoPE
    transpose (autograd through oracle.decoder.rope) of its attention
    gradients; dv is the plain attention's, bit for bit."""
    q, k, v, do = _attn_case(B, Sq, Hq, Hkv, hd, 3 * Sq)
    qg, kg, vg, dog = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o = torch.empty(B, Sq, Hq, hd, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device="cuda")
    lsq.lsq_attention_fwd(qg, kg, vg, o, lse, B, Sq, Hq, Hkv, hd)
    table = lsq.rope_table(theta, Sq, hd)
    ws = torch.empty(lsq.lsq_attention_bwd_workspace_size(B, Sq, Hq), dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.empty_like(o), torch.empty_like(kg), torch.empty_like(vg)
    lsq.lsq_attention_bwd_ex(qg, kg, vg, o, lse, dog, dq, dk, dv, B, Sq, Hq, Hkv, hd, table, ws)
    dq0, dk0, dv0 = torch.empty_like(o), torch.empty_like(kg), torch.empty_like(vg)
    lsq.lsq_attention_bwd(qg, kg, vg, o, lse, dog, dq0, dk0, dv0, B, Sq, Hq, Hkv, hd, ws)
    torch.cuda.synchronize()
    assert torch.equal(dv, dv0)
    bnd = attention_bounds(q, k, v, do)

    def rope_t(g):   # the oracle's RoPE transpose of g (autograd through its forward rotation)
        z = torch.zeros_like(g, dtype=F64).requires_grad_(True)
        return torch.autograd.grad(D.rope(z, theta), z, grad_outputs=g.to(F64))[0]

    h = hd // 2
    for name, got, g, b in (("dq rope", dq, bnd["dq"], bnd["b_dq"]), ("dk rope", dk, bnd["dk"], bnd["b_dk"])):
        ref = rope_t(g)
        # the unrotated gradient's bound carried through the rotation (|cos|, |sin| <= 1: column i
        # takes the bounds of i and its partner), plus one more rounding of the rotated value
        w = torch.cat([b[..., :h] + b[..., h:], b[..., h:] + b[..., :h]], dim=-1)
        bound = w + 2.0 ** -8 * ref.abs()
        assert_within_bound(_np(got), ref.numpy(), bound.numpy(), what=name)
