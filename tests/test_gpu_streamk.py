"""Stream-K scheduling of the fused NF4 GEMM, on the GPU.

With a workspace that has room for it, a GEMM whose 512 x 256 tiles do not
fill whole rounds of the SM-pair clusters splits its weight blocks into one
contiguous range per cluster; a range that ends inside a tile leaves an fp32
partial that the cluster finishing the tile adds.  The shapes below are
chosen so that this path runs (M >= 512, at least 8 weight blocks, about 38
tiles for 74 clusters: ranges of about 8 blocks in 16-block tiles, so tiles
are cut into two and three pieces and some ranges lie wholly inside a tile):

* forward and dX (one and several segments, ragged M) against the fp64 oracle;
* bit-identical results run to run (the partials are added in cluster order);
* LoRA with B = 0 equals the plain linear bit for bit (the LoRA block sits in
  the piece that finishes each tile, after the weight blocks, on both sides);
* the same call with whole tiles (no workspace room) agrees within the GEMM
  tolerance.

The last two cases of each test have few tiles and a long contraction (512
rows; 6 tiles of 128 weight blocks, then 2 tiles of 256): there several
clusters share each tile (by the plan's cost model five and four per tile),
so every finisher adds up to four partials, pulled into its idle stages with
bulk copies.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import lora_linear as OL
from oracle import nf4 as ON
from tolerances import assert_close

pytestmark = pytest.mark.gpu


def _f64(t):
    return t.double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t, dtype=np.float64)


def _quant(lsq, W):
    N, K = W.shape
    w = lsq.NF4Weight.empty(N, K)
    lsq.lsq_nf4_quantize(W.cuda(), w.codes, w.absmax)
    return w


def _bf16(t):
    return t.to(torch.bfloat16)


def _fwd(lsq, ws_list, x, M, A, B, r, s, ys, us, workspace):
    if len(ws_list) == 1:
        lsq.lsq_nf4_lora_fwd(ws_list[0], x, M, A[0], B[0], r, s, None, ys[0], us[0], workspace=workspace)
    else:
        lsq.lsq_nf4_lora_fwd_multi(ws_list, x, M, A, B, r, s, None, ys, us, workspace=workspace)


@pytest.mark.parametrize("M,Ns,K", [(1000, [4800], 1024), (1024, [2048, 1536, 1216], 1024), (512, [1536], 8192),
                                    (512, [512], 16384)])
def test_streamk_fwd_matches_oracle_and_is_deterministic(lsq, M, Ns, K):
    r = 16
    cases = [S.linear_case(M, n, K, r, s=1.0, seed=300 + i) for i, n in enumerate(Ns)]
    x = cases[0]["X"]
    ws_list = [_quant(lsq, c["W"]) for c in cases]
    A = [_bf16(c["A"]).cuda() for c in cases]
    B = [_bf16(c["B"]).cuda() for c in cases]
    wsz = lsq.lsq_nf4_lora_fwd_workspace_size(Ns, M, K, r)
    work = torch.zeros(wsz, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(2):
        ys = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in Ns]
        us = [torch.empty(M, r, dtype=torch.float32, device="cuda") for _ in Ns]
        _fwd(lsq, ws_list, x.cuda(), M, A, B, r, 1.0, ys, us, work)
        outs.append(ys)
    # whole tiles: a workspace with room for the rank-r part only
    base = lsq.lsq_nf4_lora_fwd_workspace_size(Ns, M, K, r) - lsq.lsq_nf4_lora_fwd_workspace_size(Ns, M, K, 0)
    small = torch.zeros(max(base, 256), dtype=torch.uint8, device="cuda")
    yw = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in Ns]
    uw = [torch.empty(M, r, dtype=torch.float32, device="cuda") for _ in Ns]
    _fwd(lsq, ws_list, x.cuda(), M, A, B, r, 1.0, yw, uw, small)
    torch.cuda.synchronize()
    for i, (c, n) in enumerate(zip(cases, Ns)):
        assert torch.equal(outs[0][i], outs[1][i])
        packed, am = ON.quantize(c["W"].float().numpy())
        Wd = ON.dequantize_f64(packed, am, n, K)
        Y, _ = OL.lora_forward(_f64(x), Wd, _f64(_bf16(c["A"])), _f64(_bf16(c["B"])), 1.0)
        assert_close(outs[0][i].float().cpu().numpy(), Y, what=f"Y[{i}] stream-K")
        assert_close(yw[i].float().cpu().numpy(), Y, what=f"Y[{i}] whole tiles")


@pytest.mark.parametrize("M,N,K", [(1000, 4800, 1024), (512, 1536, 8192)])
def test_streamk_b_zero_equals_base_bitwise(lsq, M, N, K):
    r = 16
    case = S.linear_case(M, N, K, r, seed=310)
    w = _quant(lsq, case["W"])
    x = case["X"].cuda()
    A = _bf16(case["A"]).cuda()
    Bz = torch.zeros(N, r, dtype=torch.bfloat16, device="cuda")
    work = torch.zeros(lsq.lsq_nf4_lora_fwd_workspace_size([N], M, K, r), dtype=torch.uint8, device="cuda")
    y1 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty_like(y1)
    lsq.lsq_nf4_lora_fwd(w, x, M, A, Bz, r, 2.0, None, y1, None, workspace=work)
    lsq.lsq_nf4_lora_fwd(w, x, M, None, None, 0, 0.0, None, y2, None, workspace=work)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("M,Ns,K", [(1000, [1024], 4800), (1024, [512, 256, 256], 4800), (512, [4096, 4096], 1536),
                                    (512, [16384], 512)])
def test_streamk_dx_matches_oracle_and_is_deterministic(lsq, M, Ns, K):
    r = 16
    cases = [S.linear_case(M, n, K, r, s=1.0, seed=320 + i) for i, n in enumerate(Ns)]
    x = cases[0]["X"].cuda()
    ws_list = [_quant(lsq, c["W"]) for c in cases]
    A = [_bf16(c["A"]).cuda() for c in cases]
    B = [_bf16(c["B"]).cuda() for c in cases]
    dys = [c["dY"].cuda() for c in cases]
    us = [torch.from_numpy((_f64(cases[0]["X"]) @ _f64(_bf16(c["A"])).T).astype(np.float32)).cuda() for c in cases]
    work = torch.zeros(lsq.lsq_nf4_lora_bwd_workspace_size(Ns, M, K, r), dtype=torch.uint8, device="cuda")
    dxs = []
    for _ in range(2):
        dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
        dA = [torch.empty(r, K, dtype=torch.float32, device="cuda") for _ in Ns]
        dB = [torch.empty(n, r, dtype=torch.float32, device="cuda") for n in Ns]
        if len(Ns) == 1:
            lsq.lsq_nf4_lora_bwd(ws_list[0], x, dys[0], M, A[0], B[0], r, 1.0, us[0], dx, dA[0], dB[0], 0, work)
        else:
            lsq.lsq_nf4_lora_bwd_multi(ws_list, x, dys, M, A, B, r, 1.0, us, dx, dA, dB, 0, work)
        dxs.append(dx)
    torch.cuda.synchronize()
    assert torch.equal(dxs[0], dxs[1])
    ref = np.zeros((M, K))
    for c, n in zip(cases, Ns):
        packed, am = ON.quantize(c["W"].float().numpy())
        Wd = ON.dequantize_f64(packed, am, n, K)
        rdX, _, _, _ = OL.lora_backward(_f64(cases[0]["X"]), Wd, _f64(_bf16(c["A"])), _f64(_bf16(c["B"])), 1.0,
                                         _f64(c["dY"]))
        ref += rdX
    assert_close(dxs[0].float().cpu().numpy(), ref, what="dX stream-K")


def _two_layer_8b():
    import dataclasses
    return dataclasses.replace(S.LLAMA8B, name="llama-3.1-8b-2-layers", n_layers=2)


def _steps(tr, shape, B, Sq, n):
    losses = []
    for t in range(n):
        tr.set_ids(S.tokens(shape, B, Sq, step=t).cuda())
        tr.forward_backward()
        torch.cuda.synchronize()
        losses.append(tr.loss_dev.item())
        if t == 0:
            g0 = tr.lora.grad.clone()
        tr.optimizer_step()
    torch.cuda.synchronize()
    return losses, g0


def test_streamk_model_streamed_equals_resident_bitwise(lsq):
    """Two layers of the 8B shape at 4 x 512 tokens: every fused linear of the
    step takes the stream-K path; streamed (2 slots) and resident runs must
    still agree bit for bit."""
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    shape, B, Sq = _two_layer_8b(), 4, 512
    res = StreamedLoraTrainer(shape, B, Sq, n_slots=None, init="device")
    rl, rg = _steps(res, shape, B, Sq, 2)
    res.close()
    st = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device")
    sl, sg = _steps(st, shape, B, Sq, 2)
    st.close()
    assert sl == rl and torch.equal(sg, rg)
    assert all(np.isfinite(sl))


def test_streamk_model_dpo_zero_b_policy_is_reference_bitwise(lsq):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    shape, B, Sq = _two_layer_8b(), 4, 512
    tr = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device")
    lp = tr.lora
    for l in range(shape.n_layers):
        for n in S.LINEARS:
            lp.view(lp.op, l, n, "B").zero_()
    tr.set_ids(S.tokens(shape, B, Sq).cuda())
    tr.forward_backward_dpo(0.1)
    torch.cuda.synchronize()
    assert torch.equal(tr.pi_logp, tr.ref_logp)
    tr.close()
