"""The fused linear with a rank state kept between passes, on the GPU.

Under gradient checkpointing the layer forward runs twice with the same x,
A and B; the first call can leave the rank-r operands (s*U, the padded B,
B^T, A^T) in a state that the recompute and the backward reuse.  Everything
must stay bit-identical to the path that rebuilds them:

* forward with the state filled, and again with it reused: Y bit-identical to
  the plain forward (one and three segments, stream-K and whole tiles);
* backward reading the state: dX, dA, dB bit-identical to the plain backward;
* a whole training run with and without the state: losses and every LoRA
  gradient bit-identical;
* a missing state with r > 0 is refused.
"""
import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu


def _quant(lsq, W):
    N, K = W.shape
    w = lsq.NF4Weight.empty(N, K)
    lsq.lsq_nf4_quantize(W.cuda(), w.codes, w.absmax)
    return w


@pytest.mark.parametrize("M,Ns,K", [(1000, [4800], 1024), (256, [384, 128, 200], 320), (64, [512], 512)])
def test_state_forward_and_backward_bitwise(lsq, M, Ns, K):
    r, s = 16, 1.0
    cases = [S.linear_case(M, n, K, r, s=s, seed=400 + i) for i, n in enumerate(Ns)]
    x = cases[0]["X"].cuda()
    Ws = [_quant(lsq, c["W"]) for c in cases]
    A = [c["A"].to(torch.bfloat16).cuda() for c in cases]
    B = [c["B"].to(torch.bfloat16).cuda() for c in cases]
    wsf = torch.zeros(lsq.lsq_nf4_lora_fwd_workspace_size(Ns, M, K, r), dtype=torch.uint8, device="cuda")
    wsb = torch.zeros(lsq.lsq_nf4_lora_bwd_workspace_size(Ns, M, K, r), dtype=torch.uint8, device="cuda")
    state = torch.zeros(lsq.lsq_nf4_lora_state_size(Ns, M, K, r), dtype=torch.uint8, device="cuda")

    def outs():
        return [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in Ns]

    y0, u0 = outs(), [torch.empty(M, r, dtype=torch.float32, device="cuda") for _ in Ns]
    lsq.lsq_nf4_lora_fwd_multi(Ws, x, M, A, B, r, s, None, y0, u0, workspace=wsf)
    y1, u1 = outs(), [torch.empty(M, r, dtype=torch.float32, device="cuda") for _ in Ns]
    lsq.lsq_nf4_lora_fwd_multi_ex(Ws, x, M, A, B, r, s, None, y1, u1, state, False, workspace=wsf)
    y2 = outs()
    lsq.lsq_nf4_lora_fwd_multi_ex(Ws, x, M, A, B, r, s, None, y2, None, state, True, workspace=wsf)
    dys = [c["dY"].cuda() for c in cases]

    def bwd(with_state):
        dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
        dA = [torch.empty(r, K, dtype=torch.float32, device="cuda") for _ in Ns]
        dB = [torch.empty(n, r, dtype=torch.float32, device="cuda") for n in Ns]
        if with_state:
            lsq.lsq_nf4_lora_bwd_multi_ex(Ws, x, dys, M, A, B, r, s, None, state, dx, dA, dB, 0, wsb)
        else:
            lsq.lsq_nf4_lora_bwd_multi(Ws, x, dys, M, A, B, r, s, u0, dx, dA, dB, 0, wsb)
        return dx, dA, dB

    b0, b1 = bwd(False), bwd(True)
    torch.cuda.synchronize()
    for i in range(len(Ns)):
        assert torch.equal(y0[i], y1[i]) and torch.equal(y0[i], y2[i]), i
        assert torch.equal(u0[i], u1[i]), i
        assert torch.equal(b0[1][i], b1[1][i]) and torch.equal(b0[2][i], b1[2][i]), i
    assert torch.equal(b0[0], b1[0])


def test_state_is_required_with_an_adapter(lsq):
    M, N, K, r = 64, 128, 128, 8
    c = S.linear_case(M, N, K, r)
    w = _quant(lsq, c["W"])
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    A, B = c["A"].to(torch.bfloat16).cuda(), c["B"].to(torch.bfloat16).cuda()
    with pytest.raises(lsq.LsqError) as e:
        lsq.lsq_nf4_lora_fwd_multi_ex([w], c["X"].cuda(), M, [A], [B], r, 1.0, None, [y], None, None, False)
    assert e.value.status == 1


@pytest.mark.parametrize("shape,B,Sq", [(S.TINY_UNTIED, 2, 128)])
def test_training_with_and_without_rank_state_bitwise(lsq, shape, B, Sq):
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer
    runs = []
    for keep in (False, True):
        tr = StreamedLoraTrainer(shape, B, Sq, n_slots=2, init="device")
        tr.keep_rank_state = keep
        losses = []
        for t in range(3):
            tr.set_ids(S.tokens(shape, B, Sq, step=t).cuda())
            tr.forward_backward()
            torch.cuda.synchronize()
            losses.append(tr.loss_dev.item())
            if t == 0:
                g0 = tr.lora.grad.clone()
            tr.optimizer_step()
        torch.cuda.synchronize()
        runs.append((losses, g0))
        tr.close()
    assert runs[0][0] == runs[1][0]
    assert torch.equal(runs[0][1], runs[1][1])
