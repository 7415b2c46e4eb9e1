"""Pins for the oracle's preference loss (DPO) and sequence log-probabilities (CPU only).

The sequence log-probability against a brute-force loop; the DPO loss at zero
margin (log 2), its swap identity softplus(z) - softplus(-z) = z, its gradient
against the closed form -beta * sigmoid(-z) / P by central differences; the
whole-stack DPO loss with LoRA B = 0 (policy = reference: exactly log 2); and
the whole-stack DPO gradients against central finite differences.
"""
import math

import numpy as np
import torch

from oracle import decoder as D
from test_oracle_decoder import _tiny_model

F64 = torch.float64


def test_sequence_logprob_brute_force():
    g = torch.Generator().manual_seed(3)
    B, Sq, V = 2, 5, 7
    logits = torch.randn(B, Sq, V, generator=g, dtype=F64) * 2
    ids = torch.randint(0, V, (B, Sq), generator=g)
    got = D.sequence_logprob(logits, ids)
    for b in range(B):
        tot = 0.0
        for t in range(Sq - 1):
            row = [logits[b, t, v].item() for v in range(V)]
            mx = max(row)
            z = sum(math.exp(x - mx) for x in row)
            tot += row[int(ids[b, t + 1])] - mx - math.log(z)
        assert abs(got[b].item() - tot) < 1e-12


def test_dpo_zero_margin_is_log_two():
    pi = torch.tensor([-10.0, -12.0, -3.0, -7.5], dtype=F64)
    ref = pi - torch.tensor([0.4, 0.4, -1.0, -1.0], dtype=F64)  # same offset within each pair
    assert abs(D.dpo_loss(pi, ref, 0.1).item() - math.log(2.0)) < 1e-15


def test_dpo_swap_identity():
    pi = torch.tensor([-10.0, -12.5], dtype=F64)
    ref = torch.tensor([-11.0, -11.0], dtype=F64)
    beta = 0.1
    z = beta * ((pi[0] - ref[0]) - (pi[1] - ref[1])).item()
    swapped = D.dpo_loss(pi.flip(0), ref.flip(0), beta).item()
    assert abs((swapped - D.dpo_loss(pi, ref, beta).item()) - z) < 1e-14


def test_dpo_gradient_closed_form_by_central_differences():
    pi = torch.tensor([-10.0, -12.5, -4.0, -3.0], dtype=F64)
    ref = torch.tensor([-11.0, -11.0, -4.5, -2.0], dtype=F64)
    beta, P, h = 0.1, 2, 1e-6
    for k in range(4):
        e = torch.zeros(4, dtype=F64)
        e[k] = h
        num = (D.dpo_loss(pi + e, ref, beta).item() - D.dpo_loss(pi - e, ref, beta).item()) / (2 * h)
        i = k // 2
        z = beta * ((pi[2 * i] - ref[2 * i]) - (pi[2 * i + 1] - ref[2 * i + 1])).item()
        sig_neg = 1.0 / (1.0 + math.exp(z))
        ana = (-1.0 if k % 2 == 0 else 1.0) * beta * sig_neg / P
        assert abs(num - ana) < 1e-8, (k, num, ana)


def test_model_dpo_with_zero_b_is_log_two():
    shape, layers, emb, lora, ids = _tiny_model(5)
    for per in lora:
        for t in per.values():
            t["B"].zero_()
    ids = torch.cat([ids, ids.flip(1)], 0)  # 4 sequences = 2 pairs
    loss, grads, pi, ref = D.model_dpo_loss_and_grads(ids, layers, emb, lora, shape)
    assert torch.equal(pi, ref)
    assert loss == math.log(2.0)
    for per in grads:  # B = 0 leaves no path to A
        for t in per.values():
            assert float(t["A"].abs().max()) == 0.0


def test_model_dpo_gradients_match_central_differences():
    shape, layers, emb, lora, ids = _tiny_model(6)
    ids = torch.cat([ids, ids.flip(1)], 0)
    loss, grads, _, _ = D.model_dpo_loss_and_grads(ids, layers, emb, lora, shape, beta=0.5)

    def f():
        with torch.no_grad():
            ref = D.sequence_logprob(D.model_logits(ids, layers, emb, lora, shape, 0.0), ids)
            pi = D.sequence_logprob(D.model_logits(ids, layers, emb, lora, shape, shape.s), ids)
            return D.dpo_loss(pi, ref, 0.5).item()

    assert abs(f() - loss) < 1e-12
    rng = np.random.default_rng(1)
    h = 1e-6
    for l in range(shape.n_layers):
        for name in ("q", "o", "up", "down"):
            for ab in ("A", "B"):
                P = lora[l][name][ab]
                num, ana = [], []
                for _ in range(2):
                    i = tuple(int(rng.integers(0, s)) for s in P.shape)
                    old = P[i].item()
                    P[i] = old + h
                    fp = f()
                    P[i] = old - h
                    fm = f()
                    P[i] = old
                    num.append((fp - fm) / (2 * h))
                    ana.append(grads[l][name][ab][i].item())
                num, ana = np.array(num), np.array(ana)
                assert np.linalg.norm(num - ana) <= 1e-6 * np.linalg.norm(ana) + 1e-10, (l, name, ab, num, ana)
