"""Pins for the oracle's decoder stack, loss and optimizer (CPU only).

Closed forms and special cases (S = 1 attention, RoPE at position 0, RoPE as a
complex rotation, unit RMS, uniform logits), brute-force attention on a tiny
case, causality, central finite differences of the whole-stack loss, and the
AdamW closed form for a constant gradient.
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import decoder as D
from oracle import train as T

F64 = torch.float64


def test_rmsnorm_unit_rms():
    x = torch.randn(4, 7, 32, dtype=F64) * 3
    y = D.rmsnorm(x, torch.ones(32, dtype=F64), 0.0)
    torch.testing.assert_close((y * y).mean(-1), torch.ones(4, 7, dtype=F64))


def test_rope_position_zero_identity_and_complex_rotation():
    B, Sq, H, hd, theta = 1, 6, 2, 8, 1e4
    x = torch.randn(B, Sq, H, hd, dtype=F64)
    y = D.rope(x, theta)
    torch.testing.assert_close(y[:, 0], x[:, 0])
    xc = x[..., : hd // 2].numpy() + 1j * x[..., hd // 2:].numpy()
    p = np.arange(Sq)[None, :, None, None]
    i = np.arange(hd // 2)[None, None, None, :]
    yc = xc * np.exp(1j * p * theta ** (-2.0 * i / hd))
    np.testing.assert_allclose(y[..., : hd // 2].numpy(), yc.real, atol=1e-12)
    np.testing.assert_allclose(y[..., hd // 2:].numpy(), yc.imag, atol=1e-12)


def test_attention_single_position_is_v():
    q = torch.randn(2, 1, 4, 8, dtype=F64)
    k = torch.randn(2, 1, 2, 8, dtype=F64)
    v = torch.randn(2, 1, 2, 8, dtype=F64)
    out = D.causal_gqa_attention(q, k, v)
    torch.testing.assert_close(out, v.repeat_interleave(2, dim=2))


def test_attention_brute_force_gqa():
    B, Sq, Hq, Hkv, hd = 1, 4, 4, 2, 3
    q = torch.randn(B, Sq, Hq, hd, dtype=F64)
    k = torch.randn(B, Sq, Hkv, hd, dtype=F64)
    v = torch.randn(B, Sq, Hkv, hd, dtype=F64)
    out = D.causal_gqa_attention(q, k, v)
    for h in range(Hq):
        kh = h // (Hq // Hkv)
        for i in range(Sq):
            sc = [sum(q[0, i, h, c] * k[0, j, kh, c] for c in range(hd)).item() / math.sqrt(hd) for j in range(i + 1)]
            mx = max(sc)
            e = [math.exp(t - mx) for t in sc]
            z = sum(e)
            for c in range(hd):
                want = sum(e[j] / z * v[0, j, kh, c].item() for j in range(i + 1))
                assert abs(out[0, i, h, c].item() - want) < 1e-12


def test_cross_entropy_uniform_logits_is_log_v():
    V = 37
    logits = torch.zeros(2, 5, V, dtype=F64)
    ids = torch.randint(0, V, (2, 5))
    assert abs(D.cross_entropy_next_token(logits, ids).item() - math.log(V)) < 1e-12


def _tiny_model(seed=0):
    shape = S.ModelShape("fd", 2, 16, 24, 2, 1, 11, 1e4, 1e-5, False, 2)
    g = torch.Generator().manual_seed(seed)
    layers = []
    for _ in range(shape.n_layers):
        W = {n: torch.randn(nk[0], nk[1], generator=g, dtype=F64) * 0.3 for n, nk in shape.linear_shapes().items()}
        W["ln1"] = 1 + 0.1 * torch.randn(shape.d, generator=g, dtype=F64)
        W["ln2"] = 1 + 0.1 * torch.randn(shape.d, generator=g, dtype=F64)
        layers.append(W)
    emb = {"embed": torch.randn(shape.vocab, shape.d, generator=g, dtype=F64),
           "lm_head": torch.randn(shape.vocab, shape.d, generator=g, dtype=F64) * 0.3,
           "final_norm": torch.ones(shape.d, dtype=F64)}
    lora = [{n: {"A": torch.randn(shape.r, nk[1], generator=g, dtype=F64) * 0.3,
                 "B": torch.randn(nk[0], shape.r, generator=g, dtype=F64) * 0.3}
             for n, nk in shape.linear_shapes().items()} for _ in range(shape.n_layers)]
    ids = torch.randint(0, shape.vocab, (2, 5), generator=g)
    return shape, layers, emb, lora, ids


def test_model_gradients_match_central_differences():
    shape, layers, emb, lora, ids = _tiny_model()
    loss, grads = D.model_loss_and_grads(ids, layers, emb, lora, shape)
    rng = np.random.default_rng(0)
    h = 1e-6
    for l in range(shape.n_layers):
        for name in ("q", "k", "v", "o", "gate", "up", "down"):
            for ab in ("A", "B"):
                P = lora[l][name][ab]
                idx = [tuple(int(rng.integers(0, s)) for s in P.shape) for _ in range(3)]
                num, ana = [], []
                for i in idx:
                    old = P[i].item()
                    P[i] = old + h
                    fp = D.model_loss(ids, layers, emb, lora, shape).item()
                    P[i] = old - h
                    fm = D.model_loss(ids, layers, emb, lora, shape).item()
                    P[i] = old
                    num.append((fp - fm) / (2 * h))
                    ana.append(grads[l][name][ab][i].item())
                num, ana = np.array(num), np.array(ana)
                assert np.linalg.norm(num - ana) <= 1e-6 * np.linalg.norm(ana) + 1e-10, (l, name, ab, num, ana)


def test_causality():
    shape, layers, emb, lora, ids = _tiny_model(1)
    h0 = emb["embed"][ids.long()]
    out1 = D.decoder_layer(h0, layers[0], lora[0], shape, shape.s)
    h1 = h0.clone()
    h1[:, 3] += 1.0
    out2 = D.decoder_layer(h1, layers[0], lora[0], shape, shape.s)
    torch.testing.assert_close(out1[:, :3], out2[:, :3], rtol=0, atol=1e-14)
    assert (out1[:, 3] - out2[:, 3]).abs().max() > 1e-3


def test_loss_at_init_near_log_vocab():
    shape = S.TINY
    layers = [S.layer_weights(shape, l) for l in range(shape.n_layers)]
    emb = S.embeddings(shape)
    lora = [{n: {ab: t[ab] for ab in ("A", "B")} for n, t in per.items()} for per in S.lora_init(shape)]
    ids = S.tokens(shape, 1, 16)
    losses, _, _ = T.train(shape, layers, emb, lora, [ids])
    assert abs(losses[0] - math.log(shape.vocab)) < 0.05 * math.log(shape.vocab)


def test_adamw_constant_gradient_closed_form():
    p = torch.tensor([1.0, -2.0, 0.5], dtype=F64)
    g = torch.tensor([0.3, -1e-3, 2.0], dtype=F64)
    m = torch.zeros(3, dtype=F64)
    v = torch.zeros(3, dtype=F64)
    lr, eps = 1e-2, 1e-8
    want = p.clone()
    for t in range(1, 6):
        p, m, v = D.adamw(p, g, m, v, t, lr=lr, eps=eps)
        # with a constant gradient both bias-corrected moments are exact: m^ = g, v^ = g^2
        want = want - lr * g / (g.abs() + eps)
        torch.testing.assert_close(p, want, rtol=1e-12, atol=1e-14)
