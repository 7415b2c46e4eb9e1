"""The allocation-free backward entry point against the workspace one.

lsq_nf4_lora_bwd_noalloc serves callers that cannot allocate device memory
(a host framework that owns the whole pool and hands out no allocator, a
hard per-process memory cap): it takes the same inputs and outputs as
lsq_nf4_lora_bwd but uses a scratch array the library holds itself.  Calls in
a row with different sizes must give what the workspace entry point gives:
within the tolerance the other backward tests use and, since both take the
same plan up to the 8B shapes (the array holds the dX GEMM's stream-K
partials too), bit for bit.  The first call covers the 8B down projection at
2048 tokens, the largest single linear of the 8B step (15.9 MiB of scratch
besides the stream-K partials).  This file is collected last so that a
failure here leaves every other test already run.
"""
import numpy as np
import pytest
import torch

import synthetic as S
from tolerances import assert_close

pytestmark = pytest.mark.gpu


def _case(lsq, M, N, K, r, seed):
    c = S.linear_case(M, N, K, r, s=16.0 / r, seed=seed)
    w = lsq.NF4Weight.empty(N, K)
    lsq.lsq_nf4_quantize(c["W"].cuda(), w.codes, w.absmax)
    A = c["A"].to(torch.bfloat16).cuda()
    B = c["B"].to(torch.bfloat16).cuda()
    x, dy = c["X"].cuda(), c["dY"].cuda()
    u = torch.empty(M, r, dtype=torch.float32, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    lsq.lsq_nf4_lora_fwd(w, x, M, A, B, r, c["s"], None, y, u)
    return w, x, dy, A, B, u, c["s"]


def _outs(M, N, K, r):
    return (torch.empty(M, K, dtype=torch.bfloat16, device="cuda"),
            torch.empty(r, K, dtype=torch.float32, device="cuda"),
            torch.empty(N, r, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("sizes", [[(2048, 4096, 14336, 16), (200, 512, 1024, 16), (64, 328, 576, 8)]])
def test_noalloc_bwd_matches_workspace_bwd(lsq, sizes):
    for call, (M, N, K, r) in enumerate(sizes):          # calls in a row, each size once
        w, x, dy, A, B, u, s = _case(lsq, M, N, K, r, seed=40 + call)
        dx0, dA0, dB0 = _outs(M, N, K, r)
        ws = torch.empty(lsq.lsq_nf4_lora_bwd_workspace_size([N], M, K, r), dtype=torch.uint8, device="cuda")
        lsq.lsq_nf4_lora_bwd(w, x, dy, M, A, B, r, s, u, dx0, dA0, dB0, 0, ws)
        dx1, dA1, dB1 = _outs(M, N, K, r)
        lsq.lsq_nf4_lora_bwd_noalloc(w, x, dy, M, A, B, r, s, u, dx1, dA1, dB1, 0)
        torch.cuda.synchronize()
        assert_close(dx1.float().cpu().numpy(), dx0.float().cpu().numpy().astype(np.float64), what="dX")
        assert_close(dA1.cpu().numpy(), dA0.cpu().numpy().astype(np.float64), what="dA")
        assert_close(dB1.cpu().numpy(), dB0.cpu().numpy().astype(np.float64), what="dB")
        assert torch.equal(dx1, dx0) and torch.equal(dA1, dA0) and torch.equal(dB1, dB0), (M, N, K, r)
        del ws


def test_noalloc_rejects_sizes_beyond_its_scratch(lsq):
    cap = lsq.lsq_nf4_lora_bwd_noalloc_max_scratch()
    # the workspace query is the scratch the call needs plus at most ~38 MB of stream-K
    # partials, so a size whose query exceeds twice the array needs more than the array
    M = 1 << 16
    while lsq.lsq_nf4_lora_bwd_workspace_size([64], M, 64, 16) <= 2 * cap:
        M *= 2
    w = lsq.NF4Weight.empty(64, 64)
    t = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    f = torch.empty(64, dtype=torch.float32, device="cuda")
    with pytest.raises(lsq.LsqError) as e:
        lsq.lsq_nf4_lora_bwd_noalloc(w, t, t, M, t, t, 16, 1.0, f, t, f, f, 0)
    assert e.value.status == 1 and "scratch" in str(e.value)
