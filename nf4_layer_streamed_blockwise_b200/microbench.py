"""Per-kernel timing of the fused NF4-LoRA GEMMs at one stack's layer shapes.

    python -m nf4_layer_streamed_blockwise_b200.microbench [--shape llama-3.1-8b] [--batch 4] [--seq 512]
        [--iters 20] [--only fwd_qkv,...]

For every linear group of a decoder layer (q/k/v fused, o, gate/up fused,
down) it times the forward call (all its kernels), the backward call, the dX
GEMM alone (no adapter), the causal attention of one layer (forward; backward
counted as 2.5x the forward FLOPs), and the lm_head GEMMs,
with CUDA events around each launch and a 256 MB L2 flush between launches;
prints one JSON line per kernel (median ms, TFLOP/s, fraction of the
measured bf16 peak).  Inputs are random; only timing is reported.
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


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["bf16_tflops"], "measured"
    except Exception:
        return 1590.0, "fallback"


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
    a = ap.parse_args()
    sh = S.SHAPES[a.shape]
    M, r, s = a.batch * a.seq, sh.r, sh.s
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
        dys = [torch.randn(M, n, **bf) for n in ns]
        dx = torch.empty(M, K, **bf)
        dA = [torch.empty(r, K, dtype=torch.float32, device="cuda") for _ in ns]
        dB = [torch.empty(n, r, dtype=torch.float32, device="cuda") for n in ns]
        ws = torch.empty(L.lsq_nf4_lora_bwd_workspace_size(ns, M, K, r), dtype=torch.uint8, device="cuda")
        run(f"bwd_{g}", fl, lambda: L.lsq_nf4_lora_bwd_multi(Ws, x, dys, M, A, B, r, s, us, dx, dA, dB, 0, ws))
        fl0 = sum(2.0 * M * n * K for n in ns)
        run(f"dx_{g}", fl0, lambda: L.lsq_nf4_lora_bwd_multi(Ws, x, dys, M, None, None, 0, 0.0, None, dx, None, None,
                                                                0, None))
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
