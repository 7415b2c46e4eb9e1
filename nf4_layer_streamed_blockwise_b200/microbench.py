"""Per-kernel timing of the fused NF4-LoRA GEMMs at one stack's layer shapes.

    python -m nf4_layer_streamed_blockwise_b200.microbench [--shape llama-3.1-8b] [--batch 4] [--seq 512]
        [--iters 20] [--only fwd_qkv,...] [--hbm]

For every linear group of a decoder layer (q/k/v fused, o, gate/up fused,
down) it times the forward call (all its kernels), the backward call, the dX
GEMM alone (no adapter), the causal attention of one layer (forward; backward
counted as 2.5x the forward FLOPs), and the lm_head GEMMs,
with CUDA events around each launch and a 256 MB L2 flush between launches;
prints one JSON line per kernel (median ms, TFLOP/s, fraction of the
measured bf16 peak).  With --hbm it times the memory-bound kernels instead
(RMSNorm, RoPE, SwiGLU, cross entropy, AdamW, NF4 quantise / dequantise, the
double-quantised absmax expansion, the embedding gather) at the same layer
sizes and reports their algorithmic bytes (each input read once, each output
written once) per second against the measured HBM bandwidth.  Inputs are
random; only timing is reported.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics

import torch

import synthetic as S
from . import lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def peaks(key="bf16_tflops", fallback=1590.0):
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d[key], "measured"
    except Exception:
        return fallback, "fallback"


def timer(iters, flush):
    """fn -> median ms over `iters` launches, L2 flushed before each, after one warm-up call."""
    def run(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(iters):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)
    return run


def hbm_kernels(sh, M, iters, only=None):
    """The memory-bound kernels of a training step at one stack's sizes."""
    peak, src = peaks("hbm_gbs", 6650.0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    t = timer(iters, flush)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    d, f, V = sh.d, sh.f, sh.vocab
    out = []

    def run(name, nbytes, fn):
        if only and name not in only:
            return
        ms = t(fn)
        gbs = nbytes / (ms * 1e-3) / 1e9
        line = {"kernel": name, "M": M, "bytes": nbytes, "ms": ms, "gbs": gbs, "frac_of_hbm": gbs / peak,
                "peak_gbs": peak, "peak_source": f"{src} hbm_gbs"}
        out.append(line)
        print(json.dumps(line), flush=True)

    x, y, dy, res, dres = (torch.randn(M, d, **bf) for _ in range(5))
    g = torch.ones(d, **bf)
    rstd = torch.empty(M, **f32)
    run("rmsnorm_fwd", 4 * M * d + 4 * M + 2 * d, lambda: L.lsq_rmsnorm_fwd(x, g, y, rstd, M, d, sh.eps))
    run("rmsnorm_bwd", 8 * M * d + 4 * M + 2 * d, lambda: L.lsq_rmsnorm_bwd(dy, x, g, rstd, res, dres, M, d))
    Bt = M // 512 if M % 512 == 0 else 1
    Sq = M // Bt
    run("rope_q", 4 * M * d, lambda: L.lsq_rope(x, Bt, Sq, sh.n_q, sh.hd, sh.theta, 0))
    del x, y, dy, res, dres
    n = M * f
    gg, uu, mm = (torch.randn(n, **bf) for _ in range(3))
    run("swiglu_fwd", 6 * n, lambda: L.lsq_swiglu_fwd(gg, uu, mm, n))
    run("swiglu_bwd", 10 * n, lambda: L.lsq_swiglu_bwd(mm, gg, uu, gg, uu, n))
    del gg, uu, mm
    logits = torch.randn(M, V, **f32)
    ids = torch.randint(0, V, (M,), dtype=torch.int32, device="cuda")
    loss = torch.zeros(1, **f32)
    dl = torch.empty(M, V, **bf)
    wsx = torch.empty(L.lsq_xent_workspace_size(M), dtype=torch.uint8, device="cuda")
    run("xent_fwd_bwd", 6 * M * V + 4 * M, lambda: L.lsq_xent_fwd_bwd(logits, ids, Bt, Sq, V, loss, dl, wsx))
    del logits, dl
    table = torch.randn(V, d, **bf)
    h = torch.empty(M, d, **bf)
    run("embed_gather", 4 * M * d + 4 * M, lambda: L.lsq_embed_gather(ids, table, h, M, d, V))
    del table, h
    lora_n = sum(sh.r * (k + nn) for nn, k in sh.linear_shapes().values()) * sh.n_layers
    p, gr, m1, v1 = (torch.randn(lora_n, **f32) for _ in range(4))
    v1.abs_()
    pb = torch.empty(lora_n, **bf)
    run("adamw", 30 * lora_n, lambda: L.lsq_adamw_step(p, gr, m1, v1, pb, lora_n, 1, 2e-5, 0.9, 0.999, 1e-8, 0.0))
    del p, gr, m1, v1, pb
    w = torch.randn(f, d, **bf) * 0.02
    q = L.NF4Weight.empty(f, d)
    run("nf4_quantize", 2 * f * d + f * d // 2 + f * d // 16, lambda: L.lsq_nf4_quantize(w, q.codes, q.absmax))
    wd = torch.empty(f, d, **bf)
    run("nf4_dequantize", f * d // 2 + f * d // 16 + 2 * f * d, lambda: L.lsq_nf4_dequantize(q, wd))
    nb = f * d // 64
    c8 = torch.empty(nb, dtype=torch.uint8, device="cuda")
    pp = torch.empty((nb + 255) // 256 * 2, **f32)
    L.lsq_absmax_double_quantize(q.absmax, nb, c8, pp)
    am = torch.empty(nb, **f32)
    run("absmax_expand", nb + 8 * ((nb + 255) // 256) + 4 * nb, lambda: L.lsq_absmax_expand(c8, pp, nb, am))
    return out


def quantized(n, k, stream):
    w = L.NF4Weight.empty(n, k)
    L.lsq_nf4_quantize(S.device_normal_bf16((n, k), 0.02, 0, stream), w.codes, w.absmax)
    return w


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--shape", default="llama-3.1-8b")
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--seq", type=int, default=512)
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--only", default="")
    ap.add_argument("--hbm", action="store_true", help="the memory-bound kernels (GB/s against HBM)")
    a = ap.parse_args()
    sh = S.SHAPES[a.shape]
    M, r, s = a.batch * a.seq, sh.r, sh.s
    if a.hbm:
        return hbm_kernels(sh, M, a.iters, set(a.only.split(",")) if a.only else None)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    peak, src = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    groups = {"qkv": ([sh.d, sh.kv, sh.kv], sh.d), "o": ([sh.d], sh.d), "gateup": ([sh.f, sh.f], sh.d),
              "down": ([sh.d], sh.f)}
    only = set(a.only.split(",")) if a.only else None
    results = []

    def run(name, flops, fn):
        if only and name not in only:
            return
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(a.iters):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ms = statistics.median(ts)
        tf = flops / (ms * 1e-3) / 1e12
        line = {"kernel": name, "M": M, "ms": ms, "tflops": tf, "frac_of_peak": tf / peak,
                "peak_tflops": peak, "peak_source": f"{src} bf16_tflops (burst)"}
        results.append(line)
        print(json.dumps(line), flush=True)

    for g, (ns, K) in groups.items():
        Ws = [quantized(n, K, 100 + i) for i, n in enumerate(ns)]
        x = torch.randn(M, K, **bf)
        A = [torch.randn(r, K, **bf) * 0.02 for _ in ns]
        B = [torch.randn(n, r, **bf) * 0.01 for n in ns]
        ys = [torch.empty(M, n, **bf) for n in ns]
        us = [torch.empty(M, r, dtype=torch.float32, device="cuda") for _ in ns]
        fl = sum(2.0 * M * n * K + 2.0 * M * r * K + 2.0 * M * n * r for n in ns)
        wsf = torch.empty(L.lsq_nf4_lora_fwd_workspace_size(ns, M, K, r), dtype=torch.uint8, device="cuda")
        run(f"fwd_{g}", fl, lambda: L.lsq_nf4_lora_fwd_multi(Ws, x, M, A, B, r, s, None, ys, us, workspace=wsf))
        if g in ("o", "down"):   # as in the decoder layer: the residual stream added in the epilogue
            res = [torch.randn(M, n, **bf) for n in ns]
            run(f"fwd_{g}_res", fl, lambda: L.lsq_nf4_lora_fwd_multi(Ws, x, M, A, B, r, s, res, ys, us, workspace=wsf))
            del res
        if g == "qkv" and sh.hd in (64, 128, 256):   # the same call with q and k rotated in the epilogue
            table = L.rope_table(sh.theta, a.seq, sh.hd)
            run("fwd_qkv_rope", fl, lambda: L.lsq_nf4_lora_fwd_multi_ex2(Ws, x, M, A, B, r, s, None, ys, us, None,
                                                                          False, (table, a.seq, sh.hd, 0b011),
                                                                          workspace=wsf))
        dys = [torch.randn(M, n, **bf) for n in ns]
        dx = torch.empty(M, K, **bf)
        dA = [torch.empty(r, K, dtype=torch.float32, device="cuda") for _ in ns]
        dB = [torch.empty(n, r, dtype=torch.float32, device="cuda") for n in ns]
        ws = torch.empty(L.lsq_nf4_lora_bwd_workspace_size(ns, M, K, r), dtype=torch.uint8, device="cuda")
        run(f"bwd_{g}", fl, lambda: L.lsq_nf4_lora_bwd_multi(Ws, x, dys, M, A, B, r, s, us, dx, dA, dB, 0, ws))
        fl0 = sum(2.0 * M * n * K for n in ns)
        run(f"dx_{g}", fl0, lambda: L.lsq_nf4_lora_bwd_multi(Ws, x, dys, M, None, None, 0, 0.0, None, dx, None, None,
                                                                0, None))
        # the calls of a training step's backward half: the layer's first forward leaves a rank state
        # (s*U and the padded LoRA operands), which its checkpoint recompute (rfwd: the fused GEMM
        # alone, with the residual or RoPE the layer uses) and its backward (sbwd: G, dX, dA, dB) reuse
        st = torch.zeros(L.lsq_nf4_lora_state_size(ns, M, K, r), dtype=torch.uint8, device="cuda")
        resr = [torch.randn(M, n, **bf) for n in ns] if g in ("o", "down") else None
        roper = ((L.rope_table(sh.theta, a.seq, sh.hd), a.seq, sh.hd, 0b011)
                 if g == "qkv" and sh.hd in (64, 128, 256) else None)
        L.lsq_nf4_lora_fwd_multi_ex2(Ws, x, M, A, B, r, s, resr, ys, None, st, False, roper, workspace=wsf)
        flr = sum(2.0 * M * n * K + 2.0 * M * n * r for n in ns)
        run(f"rfwd_{g}", flr, lambda: L.lsq_nf4_lora_fwd_multi_ex2(Ws, x, M, A, B, r, s, resr, ys, None, st, True, roper,
                                                                   workspace=wsf))
        run(f"sbwd_{g}", fl, lambda: L.lsq_nf4_lora_bwd_multi_ex(Ws, x, dys, M, A, B, r, s, None, st, dx, dA, dB, 0,
                                                                  ws))
        del st, resr, roper
        del Ws, x, A, B, ys, us, dys, dx, dA, dB, ws, wsf
    # causal GQA attention of one layer (the batch's sequences), forward and backward
    Hq, Hkv, hd, Bt, Sq = sh.n_q, sh.n_kv, sh.hd, a.batch, a.seq
    q, o, do = (torch.randn(Bt * Sq, Hq * hd, **bf) for _ in range(3))
    k, v = (torch.randn(Bt * Sq, Hkv * hd, **bf) for _ in range(2))
    lse = torch.empty(Bt * Hq * Sq, dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsa = torch.empty(L.lsq_attention_bwd_workspace_size(Bt, Sq, Hq), dtype=torch.uint8, device="cuda")
    fa = 4.0 * Bt * Hq * Sq * Sq * hd / 2  # causal: half of the two S x S x hd products
    run("attn_fwd", fa, lambda: L.lsq_attention_fwd(q, k, v, o, lse, Bt, Sq, Hq, Hkv, hd))
    run("attn_bwd", 2.5 * fa, lambda: L.lsq_attention_bwd(q, k, v, o, lse, do, dq, dk, dv, Bt, Sq, Hq, Hkv, hd, wsa))
    del q, o, do, k, v, lse, dq, dk, dv, wsa
    hn = torch.randn(M, sh.d, **bf)
    E = torch.randn(sh.vocab, sh.d, **bf) * 0.02
    logits = torch.empty(M, sh.vocab, dtype=torch.float32, device="cuda")
    run("lm_head_fwd", 2.0 * M * sh.vocab * sh.d, lambda: L.lsq_dense_gemm(hn, E, logits, M, sh.vocab, sh.d, 0, 1))
    dl = torch.randn(M, sh.vocab, **bf)
    run("lm_head_dx", 2.0 * M * sh.vocab * sh.d, lambda: L.lsq_dense_gemm(dl, E, hn, M, sh.d, sh.vocab, 1, 0))
    return results


if __name__ == "__main__":
    main()
