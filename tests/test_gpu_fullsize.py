"""Parity at the full 8B and 32B sizes, in the launch configuration bench.py times.

Every fused linear of one 8B and one 32B decoder layer at 2048 tokens (q/k/v,
o, gate/up, down), the 8B lm_head GEMMs and the attention of 4 x 512 tokens
(32 / 8 and 40 / 8 heads) run exactly as in a training step (stream-K
workspace, rank state filled by the forward and reused by the recompute and
the backward, dA / dB beside dX).  The 32B layer's record is 274 MB, above
the 165 MiB per layer where the pages report silently wrong NF4 gradients
from the library they build on (Soup README, "Citing Soup": the repaired
wrong-gradient defect); here its gradients are checked like the 8B ones.  The fp64 oracle checks sampled outputs it can compute
one by one from its own quantisation of just the rows and blocks involved:

* Y[m, n] for sampled rows m and columns n (oracle quantises W[n, :]);
* dX[m, k] for sampled rows and one 64-wide block column k (oracle
  quantises every row's block of W there), dA[:, k] on the same block,
  dB[n, :] on the sampled columns;
* logits and the lm_head input gradient on sampled rows / columns;
* attention output and dQ / dK / dV of sampled (sequence, head) pairs.

Tolerances as the single-linear tests (tolerances.assert_close: relative
Frobenius 5e-3 and max-abs 2e-2 of the RMS on the sampled block; attention
per row).
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import decoder as D
from oracle import nf4 as ON
from tolerances import assert_close, assert_close_rows

pytestmark = pytest.mark.gpu

F64 = np.float64
M = 2048
R = 16
SCALE = 1.0


def _bf16_np(t):
    return t.to(torch.bfloat16).double().cpu().numpy()


def _wd_rows(W, rows):
    """oracle dequantised rows W[rows, :] (fp64)"""
    sub = W[rows].float().numpy()
    packed, am = ON.quantize(sub)
    return ON.dequantize_f64(packed, am, sub.shape[0], sub.shape[1])


def _wd_block(W, kb):
    """oracle dequantised block column W[:, 64 kb : 64 kb + 64] of every row (fp64)"""
    sub = W[:, 64 * kb:64 * kb + 64].float().numpy()
    packed, am = ON.quantize(sub)
    return ON.dequantize_f64(packed, am, sub.shape[0], 64)


GROUPS = {"qkv": (["q", "k", "v"], "d"), "o": (["o"], "d"), "gateup": (["gate", "up"], "d"), "down": (["down"], "f")}


@pytest.mark.parametrize("shape", ["llama-3.1-8b", "dense-32b"])
@pytest.mark.parametrize("group", list(GROUPS))
def test_fused_linear_fullsize_sampled(lsq, shape, group):
    sh = S.SHAPES[shape]
    names, kdim = GROUPS[group]
    shapes = sh.linear_shapes()
    K = sh.d if kdim == "d" else sh.f
    Ns = [shapes[n][0] for n in names]
    rng = np.random.default_rng(7)
    x = S.bf16(S.normal_f32(S.DATA_SEED, 500, (M, K)))
    Ws = [S.bf16_weight(n, K, 600 + i) for i, n in enumerate(Ns)]
    As = [torch.from_numpy(S.normal_f32(S.LORA_SEED, 700 + i, (R, K), 1.0 / math.sqrt(K))).to(torch.bfloat16)
          for i in range(len(Ns))]
    Bs = [torch.from_numpy(S.normal_f32(S.LORA_SEED, 800 + i, (n, R), 0.02)).to(torch.bfloat16)
          for i, n in enumerate(Ns)]
    dys = [S.bf16(S.normal_f32(S.DATA_SEED, 900 + i, (M, n))) for i, n in enumerate(Ns)]

    qw = []
    for W in Ws:
        w = lsq.NF4Weight.empty(W.shape[0], K)
        lsq.lsq_nf4_quantize(W.cuda(), w.codes, w.absmax)
        qw.append(w)
    ws = torch.zeros(max(lsq.lsq_nf4_lora_fwd_workspace_size(Ns, M, K, R),
                         lsq.lsq_nf4_lora_bwd_workspace_size(Ns, M, K, R)), dtype=torch.uint8, device="cuda")
    state = torch.zeros(lsq.lsq_nf4_lora_state_size(Ns, M, K, R), dtype=torch.uint8, device="cuda")
    xg, Ag, Bg = x.cuda(), [a.cuda() for a in As], [b.cuda() for b in Bs]
    y1 = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in Ns]
    y2 = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in Ns]
    lsq.lsq_nf4_lora_fwd_multi_ex(qw, xg, M, Ag, Bg, R, SCALE, None, y1, None, state, False, workspace=ws)
    lsq.lsq_nf4_lora_fwd_multi_ex(qw, xg, M, Ag, Bg, R, SCALE, None, y2, None, state, True, workspace=ws)
    dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dA = [torch.empty(R, K, dtype=torch.float32, device="cuda") for _ in Ns]
    dB = [torch.empty(n, R, dtype=torch.float32, device="cuda") for n in Ns]
    lsq.lsq_nf4_lora_bwd_multi_ex(qw, xg, [d.cuda() for d in dys], M, Ag, Bg, R, SCALE, None, state, dx, dA, dB, 0,
                                  ws)
    torch.cuda.synchronize()

    X = x.double().numpy()
    rows = np.sort(rng.choice(M, 8, replace=False))
    kb = int(rng.integers(0, K // 64))
    ks = slice(64 * kb, 64 * kb + 64)
    dx_ref = np.zeros((8, 64))
    for i, (W, n) in enumerate(zip(Ws, Ns)):
        assert torch.equal(y1[i], y2[i])                     # the recompute reuses the rank state bit for bit
        A, B, dY = _bf16_np(As[i]), _bf16_np(Bs[i]), dys[i].double().numpy()
        cols = np.sort(rng.choice(n, 128, replace=False))
        Wd = _wd_rows(W, cols)
        y_ref = X[rows] @ Wd.T + SCALE * (X[rows] @ A.T) @ B[cols].T
        assert_close(y1[i].float().cpu().numpy()[np.ix_(rows, cols)], y_ref, what=f"{group} Y[{i}]")
        Wb = _wd_block(W, kb)                                # [n, 64]
        G = dY @ B                                           # [M, r]
        dx_ref += dY[rows] @ Wb + SCALE * G[rows] @ A[:, ks]
        assert_close(dA[i].cpu().numpy()[:, ks], SCALE * G.T @ X[:, ks], what=f"{group} dA[{i}]")
        U = X @ A.T
        assert_close(dB[i].cpu().numpy()[cols], SCALE * dY[:, cols].T @ U, what=f"{group} dB[{i}]")
    assert_close(dx.float().cpu().numpy()[rows][:, ks], dx_ref, what=f"{group} dX")


def test_lm_head_fullsize_sampled(lsq):
    sh = S.LLAMA8B
    rng = np.random.default_rng(8)
    hn = S.bf16(S.normal_f32(S.DATA_SEED, 510, (M, sh.d)))
    E = S.bf16_weight(sh.vocab, sh.d, 610)
    dl = S.bf16(S.normal_f32(S.DATA_SEED, 511, (M, sh.vocab), 1e-3))
    logits = torch.empty(M, sh.vocab, dtype=torch.float32, device="cuda")
    dh = torch.empty(M, sh.d, dtype=torch.bfloat16, device="cuda")
    Eg = E.cuda()
    lsq.lsq_dense_gemm(hn.cuda(), Eg, logits, M, sh.vocab, sh.d, 0, 1)
    lsq.lsq_dense_gemm(dl.cuda(), Eg, dh, M, sh.d, sh.vocab, 1, 0)
    torch.cuda.synchronize()
    rows = np.sort(rng.choice(M, 8, replace=False))
    cols = np.sort(rng.choice(sh.vocab, 512, replace=False))
    dcols = np.sort(rng.choice(sh.d, 256, replace=False))
    H = hn[rows].double().numpy()
    assert_close(logits.cpu().numpy()[np.ix_(rows, cols)], H @ E[cols].double().numpy().T, what="logits")
    DL = dl[rows].double().numpy()
    assert_close(dh.float().cpu().numpy()[np.ix_(rows, dcols)], DL @ E[:, dcols].double().numpy(), what="dh")


@pytest.mark.parametrize("shape", ["llama-3.1-8b", "dense-32b"])
def test_attention_fullsize_sampled(lsq, shape):
    sh, B, Sq = S.SHAPES[shape], 4, 512
    Hq, Hkv, hd = sh.n_q, sh.n_kv, sh.hd
    rng = np.random.default_rng(9)
    q = S.bf16(S.normal_f32(S.DATA_SEED, 520, (B, Sq, Hq, hd)))
    k = S.bf16(S.normal_f32(S.DATA_SEED, 521, (B, Sq, Hkv, hd)))
    v = S.bf16(S.normal_f32(S.DATA_SEED, 522, (B, Sq, Hkv, hd)))
    do = S.bf16(S.normal_f32(S.DATA_SEED, 523, (B, Sq, Hq, hd)))
    o = torch.empty(B, Sq, Hq, hd, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device="cuda")
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    lsq.lsq_attention_fwd(qg, kg, vg, o, lse, B, Sq, Hq, Hkv, hd)
    dq, dk, dv = torch.empty_like(o), torch.empty_like(kg), torch.empty_like(vg)
    ws = torch.empty(lsq.lsq_attention_bwd_workspace_size(B, Sq, Hq), dtype=torch.uint8, device="cuda")
    lsq.lsq_attention_bwd(qg, kg, vg, o, lse, do.cuda(), dq, dk, dv, B, Sq, Hq, Hkv, hd, ws)
    torch.cuda.synchronize()
    group = Hq // Hkv
    for b, hk in [(0, 0), (3, Hkv - 1), (int(rng.integers(0, B)), int(rng.integers(0, Hkv)))]:
        heads = list(range(hk * group, (hk + 1) * group))
        # the oracle on one sequence and the query heads of one kv head (the whole GQA group)
        qs = q[b:b + 1, :, heads].double().requires_grad_(True)
        ks = k[b:b + 1, :, hk:hk + 1].double().requires_grad_(True)
        vs = v[b:b + 1, :, hk:hk + 1].double().requires_grad_(True)
        out = D.causal_gqa_attention(qs, ks, vs)
        out.backward(do[b:b + 1, :, heads].double())
        assert_close_rows(o[b, :, heads].float().cpu().numpy(), out[0].detach().numpy(), what=f"o b{b} kv{hk}")
        assert_close_rows(dq[b, :, heads].float().cpu().numpy(), qs.grad[0].numpy(), what=f"dq b{b} kv{hk}")
        assert_close_rows(dk[b, :, hk:hk + 1].float().cpu().numpy(), ks.grad[0].numpy(), what=f"dk b{b} kv{hk}")
        assert_close_rows(dv[b, :, hk:hk + 1].float().cpu().numpy(), vs.grad[0].numpy(), what=f"dv b{b} kv{hk}")
