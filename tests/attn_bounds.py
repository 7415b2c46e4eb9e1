"""First-order rounding-error bounds for the attention kernels' outputs.

Test infrastructure: the tolerance that the attention parity tests apply,
element by element.  It is derived from where the CUDA kernels round, not fitted
to what they produce:

* forward: the probabilities enter the P.V product as bf16 (each off by at
  most u = 2^-8 of itself), the normaliser sums the unrounded values in fp32,
  and the output is rounded to bf16 once, so
      |o^ - o|_ic <= u (|o_ic| + sum_j P_ij |v_jc|)  (+ fp32 terms);
* backward: D_i = sum_c do_ic o^_ic is formed from the bf16 forward output,
  so it inherits that output's error, |dD_i| <= sum_c |do_ic| |o^ - o|_ic;
  dS_ij = P_ij (dP_ij - D_i) is rounded to bf16 (u of itself) and carries
  P_ij |dD_i|; dQ = tau dS.K and dK = tau dS^T.Q (tau = 1/sqrt(hd)) add the
  products in fp32 and round the result to bf16 once; dV = P^T.dO takes P in
  bf16 and rounds once:
      |dq^ - dq|_ic <= u |dq_ic| + tau sum_j |ddS_ij| |k_jc|
      |dk^ - dk|_jc <= u |dk_jc| + tau sum_i |ddS_ij| |q_ic|   (summed over the GQA group)
      |dv^ - dv|_jc <= u |dv_jc| + u sum_i P_ij |do_ic|        (summed over the GQA group)
  with |ddS_ij| <= u |dS_ij| + P_ij (|dD_i| + |d dP_ij|) + eps_P P_ij |dP_ij - D_i|.

fp32 accumulation contributes at most (n + 2) 2^-24 of the matching sum of
magnitudes (n terms, the tensor cores' fp32 accumulators), and the
recomputed probabilities are off by at most eps_P = 64 x 2^-24 of themselves
(an ex2.approx of about 2^-22 relative error on scores up to a few tens).
Each bound is the worst case of errors that all point the same way; the
measured errors are random and sit well inside it (the tests record the
ratio).  A wrong index, sign or dropped term gives errors of the order of the
values themselves, far outside it.
"""
import math

import torch

U = 2.0 ** -8
EPS = 2.0 ** -24
EPS_P = 64 * EPS
F64 = torch.float64


def attention_bounds(q, k, v, do):
    """q, do [B, S, Hq, hd]; k, v [B, S, Hkv, hd] (bf16 values in fp64) ->
    dict of exact values (o, dq, dk, dv) and their bounds (b_o, b_dq, b_dk, b_dv)."""
    q, k, v, do = (t.to(F64) for t in (q, k, v, do))
    B, S, Hq, hd = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    tau = 1.0 / math.sqrt(hd)
    kk = k.repeat_interleave(g, dim=2)
    vv = v.repeat_interleave(g, dim=2)
    mask = torch.triu(torch.ones(S, S, dtype=torch.bool), diagonal=1)
    s = torch.einsum("bihd,bjhd->bhij", q, kk) * tau
    P = torch.softmax(s.masked_fill(mask, float("-inf")), dim=-1)              # [B, Hq, S, S]
    o = torch.einsum("bhij,bjhd->bihd", P, vv)
    dP = torch.einsum("bihd,bjhd->bhij", do, vv).masked_fill(mask, 0.0)
    D = (do * o).sum(-1).permute(0, 2, 1)                                        # [B, Hq, S]
    dS = P * (dP - D[..., None])
    aq, ak, av, ado = q.abs(), kk.abs(), vv.abs(), do.abs()

    PaV = torch.einsum("bhij,bjhd->bihd", P, av)
    b_o = U * (o.abs() + PaV) + EPS * (S + 2) * PaV
    dD = ((ado * b_o).sum(-1) + EPS * (hd + 2) * (ado * o.abs()).sum(-1)).permute(0, 2, 1)
    ddP = EPS * (hd + 2) * torch.einsum("bihd,bjhd->bhij", ado, av).masked_fill(mask, 0.0)
    ddS = U * dS.abs() + P * (ddP + dD[..., None]) + EPS_P * P * (dP - D[..., None]).abs()
    adS = dS.abs()

    dq = tau * torch.einsum("bhij,bjhd->bihd", dS, kk)
    b_dq = (U * dq.abs() + tau * torch.einsum("bhij,bjhd->bihd", ddS, ak)
            + EPS * (S + 2) * tau * torch.einsum("bhij,bjhd->bihd", adS, ak))

    def group_sum(x):                      # [B, S, Hq, hd] -> [B, S, Hkv, hd]
        return x.reshape(B, S, Hkv, g, hd).sum(3)

    dk = group_sum(tau * torch.einsum("bhij,bihd->bjhd", dS, q))
    mag_dk = group_sum(tau * torch.einsum("bhij,bihd->bjhd", ddS, aq)
                       + EPS * (g * S + 2) * tau * torch.einsum("bhij,bihd->bjhd", adS, aq))
    b_dk = U * dk.abs() + mag_dk
    dv = group_sum(torch.einsum("bhij,bihd->bjhd", P, do))
    PtdO = group_sum(torch.einsum("bhij,bihd->bjhd", P, ado))
    b_dv = U * dv.abs() + (U + EPS_P) * PtdO + EPS * (g * S + 2) * PtdO
    return {"o": o, "dq": dq, "dk": dk, "dv": dv, "b_o": b_o, "b_dq": b_dq, "b_dk": b_dk, "b_dv": b_dv}
