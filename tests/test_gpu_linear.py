"""GPU parity of the NF4 quantiser and the fused NF4-LoRA linear against the oracle.

Bit-exact: packed codes, absmax and dequantised bf16.  Tolerance (see
tolerances.py): forward Y, U; backward dX, dA, dB; dense GEMMs.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from oracle import lora_linear as OL
from oracle import nf4 as ON
from tolerances import assert_close

pytestmark = pytest.mark.gpu


def _oracle_quant(W_bf16: torch.Tensor):
    return ON.quantize(W_bf16.float().numpy())


def _gpu_quant(lsq, W_bf16: torch.Tensor):
    n, k = W_bf16.shape
    w = lsq.NF4Weight.empty(n, k)
    lsq.lsq_nf4_quantize(W_bf16.cuda(), w.codes, w.absmax)
    torch.cuda.synchronize()
    return w


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("shape", [(512, 512), (8, 64), (24, 576), (1000, 128)])
def test_quantize_bitexact(lsq, shape):
    W = S.bf16_weight(*shape, stream=31 + shape[0])
    w = _gpu_quant(lsq, W)
    packed, am = _oracle_quant(W)
    assert np.array_equal(w.codes.cpu().numpy(), packed)
    assert np.array_equal(w.absmax.cpu().numpy().view(np.uint32), am.reshape(-1).view(np.uint32))


def test_quantize_edge_cases_bitexact(lsq):
    # every bf16 value in [-1, 1] against absmax 1 (a block holding +1 or -1),
    # all-zero blocks, signed zeros and random absmax scales
    vals = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = ON.bf16_bits_to_f32(vals)
    f = f[np.isfinite(f) & (np.abs(f) <= 1.0)]
    n_blocks = (f.size + 62) // 63
    buf = np.zeros(n_blocks * 64, dtype=np.float32)
    for b in range(n_blocks):
        chunk = f[b * 63:(b + 1) * 63]
        buf[b * 64] = 1.0 if b % 2 == 0 else -1.0
        buf[b * 64 + 1:b * 64 + 1 + chunk.size] = chunk
    rng = np.random.default_rng(0)
    scaled = (buf.reshape(-1, 64) * ON.bf16_round(rng.uniform(1e-4, 30, size=(n_blocks, 1)).astype(np.float32)))
    extra = np.zeros((4, 64), np.float32)
    extra[1, 5] = -0.0
    extra[2, :] = -0.0
    extra[3, 7] = 3e-39                 # a subnormal
    blocks = np.concatenate([buf.reshape(-1, 64), ON.bf16_round(scaled.astype(np.float32)), extra])
    pad = (-blocks.shape[0]) % 8
    blocks = np.concatenate([blocks, np.zeros((pad, 64), np.float32)]).reshape(-1, 64 * 8)
    W = torch.from_numpy(np.ascontiguousarray(blocks)).to(torch.bfloat16)
    w = _gpu_quant(lsq, W)
    packed, am = _oracle_quant(W)
    assert np.array_equal(w.codes.cpu().numpy(), packed)
    assert np.array_equal(w.absmax.cpu().numpy().view(np.uint32), am.reshape(-1).view(np.uint32))


def test_dequantize_bitexact(lsq):
    W = S.bf16_weight(256, 512, stream=5)
    w = _gpu_quant(lsq, W)
    out = torch.empty(256, 512, dtype=torch.bfloat16, device="cuda")
    lsq.lsq_nf4_dequantize(w, out)
    packed, am = _oracle_quant(W)
    ref = ON.dequantize(packed, am, 256, 512)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), ref)


def _lora_bf16(case):
    return case["A"].to(torch.bfloat16), case["B"].to(torch.bfloat16)


def _oracle_fwd(case, packed, am, residual=None):
    N, K = case["W"].shape
    Wd = ON.dequantize_f64(packed, am, N, K)
    A, B = _lora_bf16(case)
    Y, U = OL.lora_forward(_f64(case["X"]), Wd, _f64(A), _f64(B), case["s"])
    if residual is not None:
        Y = Y + _f64(residual)
    return Y, U, Wd


@pytest.mark.parametrize("M,N,K,r", [(64, 512, 512, 8), (200, 328, 192, 16), (1, 64, 64, 3), (300, 256, 1024, 64),
                                     (130, 1536, 576, 8)])
def test_fwd_matches_oracle(lsq, M, N, K, r):
    case = S.linear_case(M, N, K, r, s=16.0 / r, seed=M + N)
    w = _gpu_quant(lsq, case["W"])
    A, B = _lora_bf16(case)
    x = case["X"].cuda()
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    u = torch.empty(M, r, dtype=torch.float32, device="cuda")
    lsq.lsq_nf4_lora_fwd(w, x, M, A.cuda(), B.cuda(), r, case["s"], None, y, u)
    torch.cuda.synchronize()
    Y, U, _ = _oracle_fwd(case, *_oracle_quant(case["W"]))
    assert_close(y.float().cpu().numpy(), Y, what="Y")
    assert_close(u.cpu().numpy(), U, rel=1e-5, max_rms=1e-4, what="U")


def test_fwd_many_tiles_per_cluster(lsq):
    """256 output tiles of 256 x 256 (8 x 32): every SM pair of the persistent
    kernel takes several, so both TMEM accumulators are reused and their
    barriers change phase more than once; M and N also leave ragged edges."""
    M, N, K, r = 1960, 8184, 128, 16
    case = S.linear_case(M, N, K, r, s=16.0 / r, seed=77)
    w = _gpu_quant(lsq, case["W"])
    A, B = _lora_bf16(case)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    u = torch.empty(M, r, dtype=torch.float32, device="cuda")
    lsq.lsq_nf4_lora_fwd(w, case["X"].cuda(), M, A.cuda(), B.cuda(), r, case["s"], None, y, u)
    torch.cuda.synchronize()
    Y, U, _ = _oracle_fwd(case, *_oracle_quant(case["W"]))
    assert_close(y.float().cpu().numpy(), Y, what="Y")
    assert_close(u.cpu().numpy(), U, rel=1e-5, max_rms=1e-4, what="U")


def test_fwd_with_residual_and_no_lora(lsq):
    M, N, K = 96, 264, 256
    case = S.linear_case(M, N, K, 8)
    w = _gpu_quant(lsq, case["W"])
    res = S.bf16(S.normal_f32(9, 9, (M, N)))
    y = res.clone().cuda()                      # residual aliases y
    lsq.lsq_nf4_lora_fwd(w, case["X"].cuda(), M, None, None, 0, 0.0, y, y, None)
    torch.cuda.synchronize()
    packed, am = _oracle_quant(case["W"])
    ref = _f64(case["X"]) @ ON.dequantize_f64(packed, am, N, K).T + _f64(res)
    assert_close(y.float().cpu().numpy(), ref, what="Y+res")


@pytest.mark.parametrize("M,N,K", [(1000, 4104, 256), (2048, 8200, 128)])
def test_fwd_residual_512_row_tiles(lsq, monkeypatch, M, N, K):
    """512-row tiles (forced) with the residual added in the staged epilogue,
    against the oracle: 34 tiles (one per cluster: the tile's whole residual
    comes in by TMA before its stores) and 132 (two per cluster for most: the
    first tile's residual a pair of chunks at a time); M and N ragged (rows
    past M and a last tile of 8 columns); the residual aliasing y gives the
    same bits."""
    monkeypatch.setenv("LSQ_NF4_TILE_ROWS", "512")
    r = 16
    case = S.linear_case(M, N, K, r, s=16.0 / r, seed=M + N + 5)
    w = _gpu_quant(lsq, case["W"])
    A, B = _lora_bf16(case)
    res = S.bf16(S.normal_f32(9, 11, (M, N)))
    x, Ag, Bg, rg = case["X"].cuda(), A.cuda(), B.cuda(), res.cuda()
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    lsq.lsq_nf4_lora_fwd(w, x, M, Ag, Bg, r, case["s"], rg, y, None)
    y2 = rg.clone()                               # residual aliases y
    lsq.lsq_nf4_lora_fwd(w, x, M, Ag, Bg, r, case["s"], y2, y2, None)
    torch.cuda.synchronize()
    Y, _, _ = _oracle_fwd(case, *_oracle_quant(case["W"]), residual=res)
    assert_close(y.float().cpu().numpy(), Y, what="Y + residual")
    assert torch.equal(y, y2)


def test_b_zero_equals_base_bitwise(lsq):
    M, N, K, r = 128, 512, 512, 8
    case = S.linear_case(M, N, K, r)
    w = _gpu_quant(lsq, case["W"])
    x = case["X"].cuda()
    A = case["A"].to(torch.bfloat16).cuda()
    Bz = torch.zeros(N, r, dtype=torch.bfloat16, device="cuda")
    y1 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty_like(y1)
    lsq.lsq_nf4_lora_fwd(w, x, M, A, Bz, r, 2.0, None, y1, None)
    lsq.lsq_nf4_lora_fwd(w, x, M, None, None, 0, 0.0, None, y2, None)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_fwd_multi_segments(lsq):
    M, K, r = 257, 320, 16
    shapes = [(384, K), (128, K), (200, K)]
    cases = [S.linear_case(M, n, K, r, s=1.0, seed=i) for i, (n, _) in enumerate(shapes)]
    x = cases[0]["X"]
    ws = [_gpu_quant(lsq, c["W"]) for c in cases]
    As = [c["A"].to(torch.bfloat16).cuda() for c in cases]
    Bs = [c["B"].to(torch.bfloat16).cuda() for c in cases]
    ys = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n, _ in shapes]
    us = [torch.empty(M, r, dtype=torch.float32, device="cuda") for _ in shapes]
    lsq.lsq_nf4_lora_fwd_multi(ws, x.cuda(), M, As, Bs, r, 1.0, None, ys, us)
    torch.cuda.synchronize()
    for i, c in enumerate(cases):
        c = dict(c, X=x)
        Y, U, _ = _oracle_fwd(c, *_oracle_quant(c["W"]))
        assert_close(ys[i].float().cpu().numpy(), Y, what=f"Y{i}")
        assert_close(us[i].cpu().numpy(), U, rel=1e-5, max_rms=1e-4, what=f"U{i}")


@pytest.mark.parametrize("M,N,K,r", [(64, 512, 512, 8), (200, 328, 192, 16), (77, 192, 576, 8), (260, 512, 1024, 64)])
def test_bwd_matches_oracle(lsq, M, N, K, r):
    case = S.linear_case(M, N, K, r, s=16.0 / r, seed=3 * M + N)
    w = _gpu_quant(lsq, case["W"])
    A, B = _lora_bf16(case)
    x, dy = case["X"].cuda(), case["dY"].cuda()
    u = torch.empty(M, r, dtype=torch.float32, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    lsq.lsq_nf4_lora_fwd(w, x, M, A.cuda(), B.cuda(), r, case["s"], None, y, u)
    dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    ws = torch.empty(lsq.lsq_nf4_lora_bwd_workspace_size([N], M, K, r), dtype=torch.uint8, device="cuda")
    lsq.lsq_nf4_lora_bwd(w, x, dy, M, A.cuda(), B.cuda(), r, case["s"], u, dx, dA, dB, 0, ws)
    torch.cuda.synchronize()
    packed, am = _oracle_quant(case["W"])
    Wd = ON.dequantize_f64(packed, am, N, K)
    rdX, rdA, rdB, _ = OL.lora_backward(_f64(case["X"]), Wd, _f64(A), _f64(B), case["s"], _f64(case["dY"]))
    assert_close(dx.float().cpu().numpy(), rdX, what="dX")
    assert_close(dA.cpu().numpy(), rdA, what="dA")
    assert_close(dB.cpu().numpy(), rdB, what="dB")
    # accumulate = 1 adds into the existing gradients
    lsq.lsq_nf4_lora_bwd(w, x, dy, M, A.cuda(), B.cuda(), r, case["s"], u, None, dA, dB, 1, ws)
    torch.cuda.synchronize()
    assert_close(dA.cpu().numpy(), 2 * rdA, what="2dA")
    assert_close(dB.cpu().numpy(), 2 * rdB, what="2dB")


def test_bwd_many_tiles_per_cluster(lsq):
    """dX over 256 tiles (8 x 32 of 256 x 256): several per SM pair; n_out = 136
    leaves a partial contraction block, M = 2000 a partial row tile."""
    M, N, K, r = 2000, 136, 8192, 16
    case = S.linear_case(M, N, K, r, s=16.0 / r, seed=78)
    w = _gpu_quant(lsq, case["W"])
    A, B = _lora_bf16(case)
    x, dy = case["X"].cuda(), case["dY"].cuda()
    u = torch.from_numpy((_f64(case["X"]) @ _f64(A).T).astype(np.float32)).cuda()
    dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dA = torch.empty(r, K, dtype=torch.float32, device="cuda")
    dB = torch.empty(N, r, dtype=torch.float32, device="cuda")
    ws = torch.empty(lsq.lsq_nf4_lora_bwd_workspace_size([N], M, K, r), dtype=torch.uint8, device="cuda")
    lsq.lsq_nf4_lora_bwd(w, x, dy, M, A.cuda(), B.cuda(), r, case["s"], u, dx, dA, dB, 0, ws)
    torch.cuda.synchronize()
    packed, am = _oracle_quant(case["W"])
    Wd = ON.dequantize_f64(packed, am, N, K)
    rdX, rdA, rdB, _ = OL.lora_backward(_f64(case["X"]), Wd, _f64(A), _f64(B), case["s"], _f64(case["dY"]))
    assert_close(dx.float().cpu().numpy(), rdX, what="dX")
    assert_close(dA.cpu().numpy(), rdA, what="dA")
    assert_close(dB.cpu().numpy(), rdB, what="dB")


def test_bwd_multi_segments_sum(lsq):
    M, K, r = 200, 256, 16
    ns = [256, 64, 192]
    cases = [S.linear_case(M, n, K, r, s=1.0, seed=10 + i) for i, n in enumerate(ns)]
    x = cases[0]["X"]
    ws_ = [_gpu_quant(lsq, c["W"]) for c in cases]
    As = [c["A"].to(torch.bfloat16) for c in cases]
    Bs = [c["B"].to(torch.bfloat16) for c in cases]
    us, dys = [], []
    for i, c in enumerate(cases):
        u = torch.from_numpy((_f64(x) @ _f64(As[i]).T).astype(np.float32)).cuda()
        us.append(u)
        dys.append(c["dY"].cuda())
    dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    dA = [torch.empty(r, K, dtype=torch.float32, device="cuda") for _ in ns]
    dB = [torch.empty(n, r, dtype=torch.float32, device="cuda") for n in ns]
    wsb = torch.empty(lsq.lsq_nf4_lora_bwd_workspace_size(ns, M, K, r), dtype=torch.uint8, device="cuda")
    lsq.lsq_nf4_lora_bwd_multi(ws_, x.cuda(), dys, M, [a.cuda() for a in As], [b.cuda() for b in Bs], r, 1.0, us, dx,
                               dA, dB, 0, wsb)
    torch.cuda.synchronize()
    rdx = 0
    for i, c in enumerate(cases):
        packed, am = _oracle_quant(c["W"])
        Wd = ON.dequantize_f64(packed, am, ns[i], K)
        d_x, d_a, d_b, _ = OL.lora_backward(_f64(x), Wd, _f64(As[i]), _f64(Bs[i]), 1.0, _f64(c["dY"]))
        rdx = rdx + d_x
        assert_close(dA[i].cpu().numpy(), d_a, what=f"dA{i}")
        assert_close(dB[i].cpu().numpy(), d_b, what=f"dB{i}")
    assert_close(dx.float().cpu().numpy(), rdx, what="dX sum")


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 1000, 576), (64, 4096, 128), (96, 512, 1000)])
@pytest.mark.parametrize("trans_b", [0, 1])
def test_dense_gemm(lsq, M, N, K, trans_b):
    a = S.bf16(S.normal_f32(7, 1, (M, K)))
    b = S.bf16(S.normal_f32(7, 2, (K, N) if trans_b else (N, K), 0.05))
    ref = _f64(a) @ (_f64(b) if trans_b else _f64(b).T)
    for out_f32 in (1, 0):
        out = torch.empty(M, N, dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
        lsq.lsq_dense_gemm(a.cuda(), b.cuda(), out, M, N, K, trans_b, out_f32)
        torch.cuda.synchronize()
        tol = 5e-5 if out_f32 else 5e-3
        assert_close(out.float().cpu().numpy(), ref, rel=tol, max_rms=2e-2, what=f"dense f32={out_f32}")


def test_bad_arguments_rejected_before_launch(lsq):
    w = lsq.NF4Weight.empty(64, 64)
    x = torch.empty(4, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lsq.LsqError) as e:
        lsq.lsq_nf4_lora_fwd(lsq.NF4Weight(w.codes, w.absmax, 64, 96), x, 4, None, None, 0, 0.0, None, y, None)
    assert e.value.status == 1
    with pytest.raises(lsq.LsqError):
        lsq.lsq_nf4_lora_fwd(w, x, 4, None, None, 65, 1.0, None, y, None)
    assert lsq.lsq_device_status() == (0, 0)


def test_bounded_wait_times_out_and_the_context_survives(lsq):
    """A wait on a flag that nothing sets runs out after its limit, records
    LSQ_ETIMEOUT (site 901) in the device status word instead of faulting,
    and the stream and context stay usable; a flag that is set passes."""
    flag = torch.zeros(1, dtype=torch.int64, device="cuda")
    torch.cuda.synchronize()
    lsq.lsq_device_status()                                # clear anything earlier tests left
    lsq.lsq_wait_flag(flag, 1, 20_000_000)                 # 20 ms, nothing sets the flag
    after = torch.ones(8, device="cuda").sum()             # queued behind the wait
    torch.cuda.synchronize()
    assert lsq.lsq_device_status() == (4, 901)
    assert after.item() == 8.0
    flag.fill_(1)
    lsq.lsq_wait_flag(flag, 1, 20_000_000)
    torch.cuda.synchronize()
    assert lsq.lsq_device_status() == (0, 0)
    with pytest.raises(lsq.LsqError) as e:
        lsq.lsq_wait_flag(flag, 1, 0)
    assert e.value.status == 1


@pytest.mark.parametrize("M,V,d,C", [(300, 3000, 512, 1024), (512, 1000, 256, 256)])
def test_dense_gemm_chunked_equals_whole_bitwise(lsq, M, V, d, C):
    """The lm_head GEMMs over vocabulary chunks (lsq_dense_gemm_ex): logits
    column blocks written with a row stride, and the input gradient's
    contraction split at the chunks, each call continuing from the fp32
    accumulator the previous left - bit-identical to the single GEMMs, which
    match the fp64 product."""
    h = S.bf16(S.normal_f32(S.DATA_SEED, 530, (M, d))).cuda()
    E = S.bf16_weight(V, d, 630).cuda()
    dl = S.bf16(S.normal_f32(S.DATA_SEED, 531, (M, V), 1e-2)).cuda()
    lg1 = torch.empty(M, V, dtype=torch.float32, device="cuda")
    lg2 = torch.full((M, V), float("nan"), dtype=torch.float32, device="cuda")
    dh1 = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    dh2 = torch.empty(M, d, dtype=torch.bfloat16, device="cuda")
    acc = torch.empty(M, d, dtype=torch.float32, device="cuda")
    lsq.lsq_dense_gemm(h, E, lg1, M, V, d, 0, 1)
    lsq.lsq_dense_gemm(dl, E, dh1, M, d, V, 1, 0)
    starts = list(range(0, V, C))
    for i, r0 in enumerate(starts):
        rows = min(C, V - r0)
        Ec = E[r0:r0 + rows].contiguous()
        lsq.lsq_dense_gemm_ex(h, d, Ec, lg2.data_ptr() + 4 * r0, V, None, M, rows, d, 0, 1)
        last = i == len(starts) - 1
        lsq.lsq_dense_gemm_ex(dl.data_ptr() + 2 * r0, V, Ec, dh2 if last else acc, d, None if i == 0 else acc,
                              M, d, rows, 1, 0 if last else 1)
    torch.cuda.synchronize()
    assert torch.equal(lg1, lg2) and torch.equal(dh1, dh2)
    Hd, Ed, Dd = h.double().cpu().numpy(), E.double().cpu().numpy(), dl.double().cpu().numpy()
    assert_close(lg2.cpu().numpy(), Hd @ Ed.T, rel=5e-5, max_rms=2e-2, what="chunked logits")
    assert_close(dh2.float().cpu().numpy(), Dd @ Ed, what="chunked dh")


@pytest.mark.parametrize("M,seq,Ns,K,hd,r,theta", [(512, 256, [512, 256, 256], 512, 128, 16, 5e5),
                                                   (384, 128, [256, 128, 128], 256, 64, 8, 1e4),
                                                   (2048, 512, [4096, 1024, 1024], 4096, 128, 16, 5e5)])
def test_fused_forward_with_rope_matches_oracle(lsq, M, seq, Ns, K, hd, r, theta):
    """q and k rotated by RoPE in the fused GEMM's epilogue (segments 0 and 1;
    v not rotated) against the oracle's linear followed by its RoPE
    (oracle.decoder.rope) on whole sequences, on up to four sampled heads of
    each segment; with the rank state and with the workspace form, bit for bit
    the same; the 8B q/k/v shape at 2048 tokens runs the stream-K tail."""
    from oracle import decoder as OD
    s = 16.0 / r
    x = S.bf16(S.normal_f32(S.DATA_SEED, 540, (M, K)))
    Ws = [S.bf16_weight(n, K, 640 + i) for i, n in enumerate(Ns)]
    As = [torch.from_numpy(S.normal_f32(S.LORA_SEED, 740 + i, (r, K), K ** -0.5)).to(torch.bfloat16) for i in range(3)]
    Bs = [torch.from_numpy(S.normal_f32(S.LORA_SEED, 840 + i, (n, r), 0.02)).to(torch.bfloat16)
          for i, n in enumerate(Ns)]
    qw = []
    for W in Ws:
        w = lsq.NF4Weight.empty(W.shape[0], K)
        lsq.lsq_nf4_quantize(W.cuda(), w.codes, w.absmax)
        qw.append(w)
    table = lsq.rope_table(theta, seq, hd)
    ws = torch.zeros(lsq.lsq_nf4_lora_fwd_workspace_size(Ns, M, K, r), dtype=torch.uint8, device="cuda")
    state = torch.zeros(lsq.lsq_nf4_lora_state_size(Ns, M, K, r), dtype=torch.uint8, device="cuda")
    xg, Ag, Bg = x.cuda(), [a.cuda() for a in As], [b.cuda() for b in Bs]
    y1 = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in Ns]
    y2 = [torch.empty(M, n, dtype=torch.bfloat16, device="cuda") for n in Ns]
    rope = (table, seq, hd, 0b011)
    lsq.lsq_nf4_lora_fwd_multi_ex2(qw, xg, M, Ag, Bg, r, s, None, y1, None, state, False, rope, workspace=ws)
    lsq.lsq_nf4_lora_fwd_multi_ex2(qw, xg, M, Ag, Bg, r, s, None, y2, None, None, False, rope, workspace=ws)
    torch.cuda.synchronize()
    X = x.double().numpy()
    rng = np.random.default_rng(11)
    for i, (W, n) in enumerate(zip(Ws, Ns)):
        assert torch.equal(y1[i], y2[i])
        heads = np.sort(rng.choice(n // hd, min(4, n // hd), replace=False))
        cols = np.concatenate([np.arange(h * hd, (h + 1) * hd) for h in heads])
        wd = W[cols].float().numpy()
        packed, am = ON.quantize(wd)
        Wd = ON.dequantize_f64(packed, am, wd.shape[0], K)
        A, B = As[i].double().numpy(), Bs[i].double().numpy()
        ref = X @ Wd.T + s * (X @ A.T) @ B[cols].T                  # [M, heads * hd]
        if i < 2:
            t = torch.from_numpy(ref).reshape(M // seq, seq, len(heads), hd)
            ref = OD.rope(t, theta).reshape(M, -1).numpy()
        assert_close(y1[i].float().cpu().numpy()[:, cols], ref, what=f"rope seg {i}")
