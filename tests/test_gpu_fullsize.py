"""Parity at the full 8B, 32B and 3B sizes, in the launch configuration bench.py times.

Every fused linear of one 8B and one 32B decoder layer at 2048 tokens and of
one Qwen2.5-3B layer at 512 tokens (q/k/v, o, gate/up, down; the 3B k and v
projections are 256 wide, one SM-pair tile), the 8B lm_head GEMMs and the tied
3B head (151936 x 2048), the attention of 4 x 512 tokens (32 / 8 and 40 / 8
heads) and of 1 x 512 tokens at 16 / 2 heads (GQA groups of 8) run exactly as
in a training step (stream-K
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
element by element within the first-order bound of its bf16 roundings,
attn_bounds.py, and relative Frobenius 5e-3).
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import decoder as D
from oracle import nf4 as ON
from attn_bounds import attention_bounds
from tolerances import assert_close, assert_within_bound

pytestmark = pytest.mark.gpu

F64 = np.float64
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


# tokens per step of each shape's workload: batch 4 x 512 (8B, 32B), batch 1 x 512 (3B)
TOKENS = {"llama-3.1-8b": 2048, "dense-32b": 2048, "qwen2.5-3b": 512}


@pytest.mark.parametrize("shape", ["llama-3.1-8b", "dense-32b", "qwen2.5-3b"])
@pytest.mark.parametrize("group", list(GROUPS))
def test_fused_linear_fullsize_sampled(lsq, shape, group):
    sh = S.SHAPES[shape]
    M = TOKENS[shape]
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


@pytest.mark.parametrize("shape", ["llama-3.1-8b", "qwen2.5-3b"])
def test_lm_head_fullsize_sampled(lsq, shape):
    """The untied 8B head (128256 x 4096) and the tied 3B embedding used as the
    head (151936 x 2048), logits and input gradient."""
    sh = S.SHAPES[shape]
    M = TOKENS[shape]
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


@pytest.mark.parametrize("shape", ["llama-3.1-8b", "dense-32b", "qwen2.5-3b"])
def test_attention_fullsize_sampled(lsq, shape):
    sh, Sq = S.SHAPES[shape], 512
    B = TOKENS[shape] // Sq
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
    for b, hk in [(0, 0), (B - 1, Hkv - 1), (int(rng.integers(0, B)), int(rng.integers(0, Hkv)))]:
        heads = list(range(hk * group, (hk + 1) * group))
        # the oracle on one sequence and the query heads of one kv head (the whole GQA group),
        # element by element within the first-order bound of the kernels' bf16 roundings
        qs, ks, vs, dos = q[b:b + 1, :, heads], k[b:b + 1, :, hk:hk + 1], v[b:b + 1, :, hk:hk + 1], do[b:b + 1, :, heads]
        bnd = attention_bounds(qs, ks, vs, dos)
        xs = [t.double().requires_grad_(True) for t in (qs, ks, vs)]
        out = D.causal_gqa_attention(*xs)
        grads = torch.autograd.grad(out, xs, grad_outputs=dos.double())
        for name, want in zip(("o", "dq", "dk", "dv"), (out.detach(), *grads)):
            assert torch.allclose(bnd[name], want, rtol=1e-9, atol=1e-12), name   # the oracle's values
        assert_within_bound(o[b:b + 1, :, heads].double().cpu().numpy(), bnd["o"].numpy(), bnd["b_o"].numpy(),
                            what=f"o b{b} kv{hk}")
        assert_within_bound(dq[b:b + 1, :, heads].double().cpu().numpy(), bnd["dq"].numpy(), bnd["b_dq"].numpy(),
                            what=f"dq b{b} kv{hk}")
        assert_within_bound(dk[b:b + 1, :, hk:hk + 1].double().cpu().numpy(), bnd["dk"].numpy(),
                            bnd["b_dk"].numpy(), what=f"dk b{b} kv{hk}")
        assert_within_bound(dv[b:b + 1, :, hk:hk + 1].double().cpu().numpy(), bnd["dv"].numpy(),
                            bnd["b_dv"].numpy(), what=f"dv b{b} kv{hk}")
