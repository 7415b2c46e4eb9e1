#!/usr/bin/env python
"""Benchmark of the streamed NF4-LoRA training step on B200.

Workload: Llama-3.1-8B-shaped stack (32 layers, hidden 4096, SwiGLU 14336,
32 q / 8 kv heads, vocab 128256, RoPE theta 5e5), random-init bf16 weights
quantised to NF4 (blocksize 64, fp32 absmax) and kept in page-locked host
RAM, streamed per decoder layer through 8 HBM slots (the top of the 2..8 range), forward 0 -> 31 and
re-streamed 31 -> 0 under gradient checkpointing; LoRA r=16 (alpha 16) on all
seven linears; AdamW on the adapters; seeded uniform token ids, seq 512.

One JSON line (rank 0):
  value         training tok/s of the whole job (batch x seq x steps x ranks / max-over-ranks time)
  e2e           same metric through the public API with token ids copied from
                pinned host memory and the loss read back every step
  roofline      fused NF4-dequant GEMM (the dominant kernel family) against the
                measured sustained bf16 tensor peak, from CUDA events around
                every launch in the timed region
  streaming     layer-copy GB/s vs the measured pinned H2D bandwidth, exposed
                copy per step (streamed - resident), peak HBM streamed vs resident
  cpu_baseline  the CPU oracle timed on a bounded sample of the same workload

`--impl reference` times that oracle alone on the same metric (see
reference_arm); under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# dram__bytes_read.sum + dram__bytes_write.sum per launch of the fused forward
# GEMM (nf4_pair_kernel<FWD>), the mean over the four calls of an 8B layer as
# the checkpoint recompute runs them (q/k/v with RoPE, o and down adding their
# residual, gate/up, at 2048 tokens: 51.1, 43.9, 197.7 and 126.3 MB), from one
# ncu capture of the kernel built from the sources whose SHA-256 prefix is
# given; the figure is reported only while those sources are unchanged (else
# traffic is null).
NCU_TRAFFIC = {("llama-3.1-8b", 2048): (104.8e6, "736a214a541a1cb0")}
TRAFFIC_SOURCES = ("nf4_layer_streamed_blockwise_b200/csrc/gemm_nf4.cu",
                   "nf4_layer_streamed_blockwise_b200/csrc/common.cuh")


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(shape, tokens):
    entry = NCU_TRAFFIC.get((shape.name, tokens))
    if entry is None or entry[1] != kernel_source_hash():
        return None
    return entry[0]


REASON_COLS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


def args_():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--shape", default="llama-3.1-8b")
    p.add_argument("--batch", type=int, default=4)
    p.add_argument("--seq", type=int, default=512)
    p.add_argument("--slots", type=int, default=8)
    p.add_argument("--no-resident", action="store_true")
    p.add_argument("--no-batch1", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--dpo", action="store_true",
                   help="DPO over pairs of sequences with the adapter-off reference on the same streamed base")
    p.add_argument("--beta", type=float, default=0.1)
    p.add_argument("--upload", default="auto", choices=["auto", "replicated", "sharded"],
                   help="with several GPUs: every rank streams whole records over its own host link "
                        "(replicated), or each rank copies 1/N of every record and an NCCL all-gather over "
                        "NVLink completes the slot (sharded; the default when N > 1)")
    p.add_argument("--source", default="ram", choices=["ram", "disk"],
                   help="where the layer records live: page-locked RAM, or a store file read by the library's "
                        "reader threads through page-locked staging buffers")
    p.add_argument("--store-path", default=None,
                   help="store file for --source disk (default: a file in the system temp directory, removed "
                        "at exit)")
    p.add_argument("--embed", default="hbm", choices=["hbm", "host"],
                   help="untied embedding table in HBM, or in page-locked host RAM read in place by the gather")
    p.add_argument("--head", default="hbm", choices=["hbm", "host"],
                   help="lm_head resident in HBM, or in page-locked host RAM streamed in vocabulary chunks of "
                        "--head-chunk rows through two HBM buffers for each of its GEMMs")
    p.add_argument("--head-chunk", type=int, default=8192)
    p.add_argument("--no-graph", action="store_true",
                   help="launch every kernel eagerly instead of replaying each step as a CUDA graph")
    p.add_argument("--absmax", default="fp32", choices=["fp32", "dq8"],
                   help="absmax format of the streamed records: fp32, or double-quantised (8-bit E4M3 codes, "
                        "blocks of 256, expanded to fp32 in HBM after each upload)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return PEAKS_FALLBACK, "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.index)],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, val in zip(REASON_COLS, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------- CPU oracle
def oracle_sample(shape, tokens: int, vocab_frac: int = 32, threads: int = None):
    """Times the fp64 oracle's training math on a bounded sample of the workload:
    one decoder layer (full width) fwd+bwd on `tokens` tokens, and the lm_head +
    cross entropy on 1/vocab_frac of the vocabulary.  Returns (seconds for the
    whole stack on `tokens` tokens by linear extrapolation, detail dict)."""
    import torch
    from oracle import decoder as OD
    if threads:
        torch.set_num_threads(threads)
    F = torch.float64
    g = torch.Generator().manual_seed(0)
    W = {n: torch.randn(nk[0], nk[1], generator=g, dtype=F) * 0.02 for n, nk in shape.linear_shapes().items()}
    W["ln1"] = torch.ones(shape.d, dtype=F)
    W["ln2"] = torch.ones(shape.d, dtype=F)
    lora = {n: {"A": (torch.randn(shape.r, nk[1], generator=g, dtype=F) / nk[1] ** 0.5).requires_grad_(True),
                "B": (torch.randn(nk[0], shape.r, generator=g, dtype=F) * 0.01).requires_grad_(True)}
            for n, nk in shape.linear_shapes().items()}
    h = torch.randn(1, tokens, shape.d, generator=g, dtype=F)
    t0 = time.perf_counter()
    out = OD.decoder_layer(h, W, lora, shape, shape.s)
    flat = [t for per in lora.values() for t in per.values()]
    torch.autograd.grad((out * out).sum(), flat)
    t_layer = time.perf_counter() - t0
    Vs = max(shape.vocab // vocab_frac, 2)
    E = torch.randn(Vs, shape.d, generator=g, dtype=F) * 0.02
    hn = torch.randn(1, tokens, shape.d, generator=g, dtype=F).requires_grad_(True)
    ids = torch.randint(0, Vs, (1, tokens), generator=g)
    t0 = time.perf_counter()
    loss = OD.cross_entropy_next_token(OD.rmsnorm(hn, torch.ones(shape.d, dtype=F), shape.eps) @ E.T, ids)
    torch.autograd.grad(loss, [hn])
    t_head = time.perf_counter() - t0
    total = shape.n_layers * t_layer + vocab_frac * t_head
    return total, {"layer_s": round(t_layer, 3), "head_slice_s": round(t_head, 3)}


def reference_arm(a):
    """The CPU oracle alone, on the same metric: each step is one bounded sample
    (see oracle_sample) extrapolated to the full stack."""
    import torch
    import synthetic as S
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    shape = S.SHAPES[a.shape]
    tokens = 128
    cores = torch.get_num_threads()
    times, walls = [], []
    for i in range(a.warmup + a.steps):
        t0 = time.perf_counter()
        t, _ = oracle_sample(shape, tokens)
        if i >= a.warmup:
            times.append(t)
            walls.append(time.perf_counter() - t0)
    sec = statistics.median(times)
    value = tokens / sec
    sample = (f"one full-width {shape.name} decoder layer fwd+bwd (fp64 oracle) on batch 1 x {tokens} tokens, "
              f"plus lm_head+CE on 1/32 of the vocabulary; each timed step is one such sample, and value is the "
              f"whole-stack rate extrapolated from it (x{shape.n_layers} layers, x32 vocabulary)")
    line = {"impl": "reference", "metric": metric_name(a, shape), "value": value,
            "unit": "tok/s", "n_gpus": a.gpus, "steps": a.steps, "warmup": a.warmup,
            "ms_per_step": statistics.median(walls) * 1e3,
            "value_basis": "extrapolated",
            "samples_run": a.warmup + a.steps,
            "extrapolated_ms_per_full_step": a.batch * a.seq / value * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(a, shape),
            "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(a, shape):
    task = (f"DPO (beta {a.beta}, {a.batch // 2} chosen/rejected pairs, reference = the base with the adapters "
            f"off, run on each layer while it is resident)") if a.dpo else "causal-LM SFT"
    store_gb = shape.n_layers * record_bytes(shape, a.absmax) / 1e9
    am = "fp32 absmax" if a.absmax == "fp32" else "double-quantised absmax: E4M3 codes, blocks of 256"
    src = "pinned host RAM" if a.source == "ram" else "a store file (disk tier: reader threads, pinned staging)"
    emb = "" if a.embed == "hbm" else ", embedding table in pinned host RAM (zero-copy gather)"
    if a.head == "host":
        emb += (f", lm_head in pinned host RAM streamed in {a.head_chunk}-row vocabulary chunks through two HBM "
                f"buffers for each of its GEMMs")
    return {"workload": f"{shape.name} shape, NF4 (bs64, {am}) base streamed from {src}{emb} through "
                        f"{a.slots} HBM slots, grad checkpointing with re-stream, LoRA r={shape.r} on all linears, "
                        f"{task}, AdamW",
            "batch": a.batch, "seq_len": a.seq, "n_slots": a.slots, "parallelism": f"dp{a.gpus}",
            "upload": a.upload if a.upload != "auto" else ("sharded" if a.gpus > 1 else "replicated"),
            "l2": f"inputs larger than L2 ({store_gb:.2f} GB of layer records streamed per pass)",
            "launch": ("eager launches" if not graph_on(a) else
                       "each step replayed as one CUDA graph (kernels, layer uploads, their events) after one "
                       "eager warm-up step; the instrumented pass runs eagerly")}


def graph_on(a):
    """Graph replay applies to the host-RAM tier without sharded uploads (the disk tier and the
    all-gather do host work in each step)."""
    return not a.no_graph and a.source == "ram" and a.upload != "sharded" and not (a.upload == "auto" and a.gpus > 1)


def record_bytes(shape, absmax="fp32"):
    """Bytes of one streamed layer record: NF4 codes + absmax of the 7 linears + 2 RMSNorm gains
    (fp32 absmax: 4 bytes per 64-weight block; double-quantised: 1 byte per block + 8 per 256 blocks)."""
    lin = shape.linear_shapes().values()
    w = sum(n * k for n, k in lin)
    if absmax == "fp32":
        am = w // 64 * 4
    else:
        am = sum(n * k // 64 + 8 * ((n * k // 64 + 255) // 256) for n, k in lin)
    return w // 2 + am + 2 * shape.d * 2


def metric_name(a, shape):
    task = "DPO train" if a.dpo else "train"
    short = {"llama-3.1-8b": "8B", "dense-32b": "32B", "qwen2.5-3b": "3B", "smollm2-135m": "135M"}.get(shape.name,
                                                                                                      shape.name)
    dq = ", double-quantised absmax" if a.absmax == "dq8" else ""
    dq += ", disk tier" if a.source == "disk" else ""
    dq += ", host embedding" if a.embed == "host" else ""
    dq += ", streamed lm_head" if a.head == "host" else ""
    return f"streamed NF4-LoRA {task} tok/s ({short} shape, seq {a.seq}{dq})"


# ---------------------------------------------------------------------------- our arm
def h2d_bandwidth(torch, nbytes=128 << 20, reps=10):
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    best = 0.0
    with torch.cuda.stream(s):
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            dst.copy_(src, non_blocking=True)
            e1.record(s)
            e1.synchronize()
            best = max(best, nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del src, dst
    return best


def step_fb(tr, a):
    """The forward/backward of one training step of the benchmarked task."""
    if getattr(a, "dpo", False):
        tr.forward_backward_dpo(a.beta)
    else:
        tr.forward_backward()


def timed_steps(torch, dist, tr, steps, ids_list, world, instrument=False, e2e=False, host_ids=None,
                loss_host=None, a=None):
    from nf4_layer_streamed_blockwise_b200 import dist as DP
    if instrument:
        tr.timeline = []
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        if e2e:
            tr.ids.copy_(host_ids[i % len(host_ids)].view(-1), non_blocking=True)
        else:
            tr.set_ids(ids_list[i % len(ids_list)])
        step_fb(tr, a)
        DP.average_gradients(tr.lora.grad, world)
        tr.optimizer_step()
        if e2e:
            loss_host[i].copy_(tr.loss_dev, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    ms = DP.max_over_ranks(e0.elapsed_time(e1), world, device="cuda")
    if dist is not None:
        dist.barrier()
    if instrument:
        tl, tr.timeline = tr.timeline, None
        return ms, tl
    return ms, None


def our_arm(a):
    """Everything runs on one non-default stream, the trainers' compute stream (stream capture
    cannot record the legacy default stream)."""
    import torch
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    with torch.cuda.stream(torch.cuda.Stream()):
        _our_arm(a)


def _our_arm(a):
    import torch
    import synthetic as S
    from nf4_layer_streamed_blockwise_b200 import lib as L
    from nf4_layer_streamed_blockwise_b200.trainer import StreamedLoraTrainer

    from nf4_layer_streamed_blockwise_b200 import dist as DP
    rank, world, local = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    rank, world, local = DP.init_from_env("nccl")
    dist = None
    if world > 1:
        import torch.distributed as dist
    shape = S.SHAPES[a.shape]
    peaks, peaks_src = load_peaks()

    h2d = h2d_bandwidth(torch)
    sharded = a.upload == "sharded" or (a.upload == "auto" and world > 1)
    a.upload = "sharded" if sharded else "replicated"
    shard = (rank, world) if sharded else None
    store_path = None
    if a.source == "disk":
        store_path = a.store_path or os.path.join(tempfile.gettempdir(), f"lsq_store_{os.getpid()}_r{rank}.bin")
        if a.store_path and world > 1:
            store_path = f"{a.store_path}.rank{rank}"
    tiers = dict(absmax=a.absmax, shard=shard, source=a.source, store_path=store_path, embed=a.embed, head=a.head,
                 head_chunk=a.head_chunk, graph=graph_on(a))
    tr = StreamedLoraTrainer(shape, a.batch, a.seq, n_slots=a.slots, init="device", **tiers)
    ids_list = [S.tokens(shape, a.batch, a.seq, step=1000 * rank + t).cuda() for t in range(4)]
    for i in range(a.warmup):
        tr.set_ids(ids_list[i % 4])
        step_fb(tr, a)
        DP.average_gradients(tr.lora.grad, world)
        tr.optimizer_step()
    tr.check_device()
    torch.cuda.reset_peak_memory_stats()
    up0, by0, re0 = tr.stats()
    hb0 = tr.head_stats()[1]
    # headline: the plain step loop (no timing events inside), clocks sampled beside it
    L.LAUNCHES[0] = 0
    clocks = ClockSampler(local)
    clocks.start()
    ms, _ = timed_steps(torch, dist, tr, a.steps, ids_list, world, a=a)
    clk = clocks.stop()
    tr.check_device()               # no bounded wait in any kernel ran out during the timed steps
    launches = L.LAUNCHES[0]
    up1, by1, re1 = tr.stats()
    hb1 = tr.head_stats()[1]
    peak_streamed = torch.cuda.max_memory_allocated()
    ms_step = ms / a.steps
    tokens = a.batch * a.seq
    value = world * tokens * a.steps / (ms * 1e-3)

    # instrumented pass (separate): CUDA events around every fused linear (per-kind
    # TFLOP/s, roofline) and around every compute-stream wait on an upload (exposed copy
    # per direction)
    L.lsq_stream_time_waits(tr.sched, 4 * shape.n_layers * a.steps)
    ms_instr, timeline = timed_steps(torch, dist, tr, a.steps, ids_list, world, instrument=True, a=a)
    wait_fwd, wait_bwd, n_waits, n_dropped = L.lsq_stream_wait_ms(tr.sched)
    L.lsq_stream_time_waits(tr.sched, 0)
    tr.check_device()
    # host time to enqueue one step on an idle GPU (the library calls of the whole step), against
    # the step's device time: a ratio near 1 means the host, not the GPU, sets the pace
    t0 = time.perf_counter()
    tr.set_ids(ids_list[0])
    step_fb(tr, a)
    tr.optimizer_step()
    host_ms = (time.perf_counter() - t0) * 1e3
    torch.cuda.synchronize()
    tr.check_device()
    kinds = {}
    for kind, flops, s0, s1 in timeline:
        d = kinds.setdefault(kind, [0.0, 0.0, 0])
        d[0] += flops
        d[1] += s0.elapsed_time(s1)
        d[2] += 1
    peak = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
    gemm = {k: {"tflops": v[0] / (v[1] * 1e-3) / 1e12, "ms_per_step": v[1] / a.steps, "launches_per_step":
                v[2] // a.steps} for k, v in kinds.items()}
    for k in gemm:
        gemm[k]["frac_of_sustained_peak"] = gemm[k]["tflops"] / peak
    dom = max(kinds, key=lambda k: kinds[k][1])
    ach = gemm[dom]["tflops"]
    all_flops = sum(v[0] for v in kinds.values())
    all_ms = sum(v[1] for v in kinds.values())

    # streaming: copy GB/s from the copy-stream events of the last uploads
    rec = tr.layout.nbytes
    up_ms = []
    for l in range(shape.n_layers):   # the instrumented (eager) pass uploaded each layer it streams
        try:
            up_ms.append(L.lsq_stream_upload_ms(tr.sched, l))
        except L.LsqError:
            pass
    copy_gbs = rec / (statistics.median(up_ms) * 1e-3) / 1e9
    streaming = {"record_bytes": rec, "uploads_per_step": (up1 - up0) / a.steps,
                 "exposed_copy_ms_fwd": wait_fwd / a.steps, "exposed_copy_ms_bwd": wait_bwd / a.steps,
                 "exposed_copy_frac": (wait_fwd + wait_bwd) / ms_instr,
                 "exposed_copy_waits_timed": n_waits, "exposed_copy_waits_dropped": n_dropped,
                 "ms_per_step_instrumented": ms_instr / a.steps,
                 "host_enqueue_ms_one_step": host_ms,
                 "h2d_bytes_per_step": (by1 - by0 + hb1 - hb0) / a.steps, "reused_per_step": (re1 - re0) / a.steps,
                 "head_h2d_bytes_per_step": (hb1 - hb0) / a.steps,
                 "copy_gbs": copy_gbs, "pinned_h2d_gbs": h2d, "copy_frac_of_link": copy_gbs / h2d,
                 "peak_hbm_gb_streamed": peak_streamed / 1e9}

    # e2e through the public API: ids from pinned host each step, loss read back
    host_ids = [t.cpu().pin_memory() for t in ids_list]
    loss_host = [torch.empty(1, dtype=torch.float32, pin_memory=True) for _ in range(a.steps)]
    ms_e2e, _ = timed_steps(torch, dist, tr, a.steps, ids_list, world, e2e=True, host_ids=host_ids,
                            loss_host=loss_host, a=a)
    tr.check_device()
    e2e = {"value": world * tokens * a.steps / (ms_e2e * 1e-3), "unit": "tok/s",
           "h2d_bytes_per_step": tokens * 4 + streaming["h2d_bytes_per_step"], "d2h_bytes_per_step": 4,
           "h2d_breakdown": {"token_ids": tokens * 4,
                             "layer_records": streaming["h2d_bytes_per_step"] - streaming["head_h2d_bytes_per_step"],
                             "lm_head_chunks": streaming["head_h2d_bytes_per_step"]},
           "last_loss": float(loss_host[-1].item())}
    store = tr
    tr.close()

    # resident run on the same store: exposed copy time and peak HBM
    if not a.no_resident:
        trr = StreamedLoraTrainer(shape, a.batch, a.seq, n_slots=None, init="device", share=store, **tiers)
        for i in range(2):
            trr.set_ids(ids_list[i % 4])
            step_fb(trr, a)
            trr.optimizer_step()
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        ms_r, _ = timed_steps(torch, dist, trr, a.steps, ids_list, world, a=a)
        trr.check_device()
        streaming["ms_per_step_resident"] = ms_r / a.steps
        # the fused linears' device time per step, resident against streamed (same instrumentation)
        ms_ri, tl_r = timed_steps(torch, dist, trr, a.steps, ids_list, world, instrument=True, a=a)
        trr.check_device()
        streaming["fused_gemm_ms_per_step_resident"] = sum(s0.elapsed_time(s1) for _, _, s0, s1 in tl_r) / a.steps
        streaming["fused_gemm_ms_per_step_streamed"] = all_ms / a.steps
        streaming["ms_per_step_resident_instrumented"] = ms_ri / a.steps
        streaming["streamed_minus_resident_ms"] = max(0.0, ms_step - ms_r / a.steps)
        streaming["peak_hbm_gb_resident"] = torch.cuda.max_memory_allocated() / 1e9
        trr.close()
        del trr

    batch1 = None
    if not a.no_batch1 and a.batch != 1 and not a.dpo:
        tr1 = StreamedLoraTrainer(shape, 1, a.seq, n_slots=a.slots, init="device", share=store, **tiers)
        ids1 = [t[:1] for t in ids_list]
        for i in range(2):
            tr1.train_step(ids1[i % 4])
        ms1, _ = timed_steps(torch, dist, tr1, a.steps, ids1, world, a=a)
        tr1.check_device()
        batch1 = {"tok_s": world * a.seq * a.steps / (ms1 * 1e-3), "ms_per_step": ms1 / a.steps}
        tr1.close()
        del tr1

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        import torch as _t
        ctoks = 128
        sec, det = oracle_sample(shape, ctoks)
        cpu = {"value": ctoks / sec, "unit": "tok/s", "cores": _t.get_num_threads(), "kind": "oracle",
               "sample": f"fp64 oracle: one full-width decoder layer fwd+bwd on 1 x {ctoks} tokens "
                         f"({det['layer_s']} s) x {shape.n_layers} layers + lm_head/CE on 1/32 of the vocabulary "
                         f"({det['head_slice_s']} s) x 32"}

    if rank == 0:
        line = {"metric": metric_name(a, shape), "value": value, "unit": "tok/s",
                "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded uniform token ids, random-init weights)",
                "config": workload_config(a, shape),
                "roofline": {"bound": "tensor",
                             "kernel": f"fused NF4-LoRA linear, {dom} (nf4_pair_kernel + lora_down_kernel)",
                             "achieved": ach, "peak": peak,
                             "unit": "TFLOP/s", "frac": ach / peak,
                             "traffic": measured_traffic(shape, a.batch * a.seq),
                             "peak_source": f"{peaks_src} bf16_tflops_sustained"},
                "fused_gemm": {"frac_of_sustained_peak": (all_flops / (all_ms * 1e-3) / 1e12) / peak,
                               "frac_of_burst_peak": (all_flops / (all_ms * 1e-3) / 1e12) /
                               peaks.get("bf16_tflops", 1650.0),
                               "share_of_step": all_ms / ms_instr, "by_kind": gemm},
                "streaming": streaming, "clocks": clk, "e2e": e2e, "gpu_launches": launches,
                "cpu_baseline": cpu}
        if batch1:
            line["batch1"] = batch1
        print(json.dumps(line), flush=True)
    if store_path and not a.store_path:
        os.remove(store_path)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    a = args_()
    if a.impl == "reference":
        reference_arm(a)
        return
    our_arm(a)


if __name__ == "__main__":
    main()
