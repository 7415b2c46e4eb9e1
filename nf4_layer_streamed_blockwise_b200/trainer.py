"""Streamed NF4-LoRA training step on one GPU, sequenced over the lsq C ABI.

The method (soup-cli 0.72.0 -> 0.72.2 diff, CHANGELOG [0.72.2] and docs
"Layer Streaming" / "NF4 streaming"; "Soup" README headline): the frozen base
is quantised once, offline, to NF4 and kept in page-locked host RAM as one
record per decoder layer; each training step streams the records through a
small ring of HBM slots, forward 0 -> L-1, and under gradient checkpointing
re-streams them L-1 -> 0 for the backward, recomputing each layer from its
saved input; the embedding and lm_head stay unquantised, on the GPU or (as the
pages plan for them) in page-locked host RAM, the head then streamed in
vocabulary chunks; the LoRA adapters are the only trained parameters
(optimizer step at the end).

This module only allocates memory (torch), builds the host store and calls
the library in order.  Every arithmetic step runs in the library's kernels.

Layer record layout (bytes, each piece 256-byte aligned): NF4 codes of
q, k, v, o, gate, up, down; then their fp32 absmax arrays in the same order;
then the two RMSNorm gains (bf16 [d] each).  With double-quantised absmax
(absmax="dq8") the record carries, instead of the fp32 arrays, each weight's
8-bit absmax codes and its (centre, scale) pairs per 256 blocks; the slot is
longer than the record by the fp32 arrays, which the scheduler expands into
after each upload (the host link carries 112.5 MB instead of 122.7 MB per 8B
layer).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch

import synthetic as S
from . import dist as DP
from . import lib as L

ALIGN = 256


def _al(n: int, a: int = ALIGN) -> int:
    return (n + a - 1) // a * a


@dataclasses.dataclass
class RecordLayout:
    """Byte offsets of one layer record (and of the fp32 absmax the kernels read,
    which lie past the record when it carries double-quantised absmax)."""
    codes: Dict[str, int]
    absmax: Dict[str, int]
    ln1: int
    ln2: int
    nbytes: int                    # bytes per record: what each upload copies
    slot_bytes: int                # bytes per HBM slot
    dq: Optional[Dict[str, tuple]] = None   # name -> (codes8 offset, params offset, n blocks)

    @staticmethod
    def of(shape: S.ModelShape, absmax: str = "fp32", record_align: int = 4096) -> "RecordLayout":
        if absmax not in ("fp32", "dq8"):
            raise ValueError(f"absmax must be 'fp32' or 'dq8', got {absmax!r}")
        off = 0
        codes, am, dq = {}, {}, {}
        lin = shape.linear_shapes()
        for name, (n, k) in lin.items():
            codes[name] = off
            off = _al(off + n * k // 2)
        for name, (n, k) in lin.items():
            nb = n * (k // 64)
            if absmax == "fp32":
                am[name] = off
                off = _al(off + nb * 4)
            else:
                c8 = off
                off = _al(off + nb)
                dq[name] = (c8, off, nb)
                off = _al(off + 8 * ((nb + 255) // 256))
        ln1 = off
        off = _al(off + shape.d * 2)
        ln2 = off
        off = _al(off + shape.d * 2)
        nbytes = _al(off, record_align)
        slot = nbytes
        if absmax == "dq8":
            for name, (n, k) in lin.items():
                am[name] = slot
                slot = _al(slot + n * (k // 64) * 4)
        return RecordLayout(codes, am, ln1, ln2, nbytes, _al(slot, record_align), dq or None)

    def expand_items(self):
        """(codes8, params, fp32 out, n blocks) per weight, for the scheduler."""
        if not self.dq:
            return []
        return [(c8, pp, self.absmax[name], nb) for name, (c8, pp, nb) in self.dq.items()]


class LayerView:
    """Typed device views into one layer record that sits in an HBM slot."""

    def __init__(self, shape: S.ModelShape, lay: RecordLayout, base: int):
        self.W = {}
        for name, (n, k) in shape.linear_shapes().items():
            self.W[name] = L.NF4Weight(base + lay.codes[name], base + lay.absmax[name], n, k)
        self.ln1 = base + lay.ln1
        self.ln2 = base + lay.ln2


class LoraParams:
    """All LoRA tensors of the stack in flat buffers: fp32 masters, grads, AdamW
    moments, and the bf16 operand copies the kernels read."""

    def __init__(self, shape: S.ModelShape, device="cuda"):
        self.shape = shape
        self.offsets = []  # per layer: {name: {"A": (off, (r, K)), "B": (off, (N, r))}}
        off = 0
        for _ in range(shape.n_layers):
            per = {}
            for name, (n, k) in shape.linear_shapes().items():
                per[name] = {"A": (off, (shape.r, k))}
                off = _al(off + shape.r * k, 64)
                per[name]["B"] = (off, (n, shape.r))
                off = _al(off + n * shape.r, 64)
            self.offsets.append(per)
        self.numel = off
        self.master = torch.zeros(off, dtype=torch.float32, device=device)
        self.grad = torch.zeros(off, dtype=torch.float32, device=device)
        self.m = torch.zeros(off, dtype=torch.float32, device=device)
        self.v = torch.zeros(off, dtype=torch.float32, device=device)
        self.op = torch.zeros(off, dtype=torch.bfloat16, device=device)
        self.step = 0

    def view(self, buf: torch.Tensor, l: int, name: str, ab: str) -> torch.Tensor:
        o, shp = self.offsets[l][name][ab]
        return buf[o:o + shp[0] * shp[1]].view(*shp)

    def init_host(self):
        """Masters from the seeded numpy streams (reproducible by the oracle)."""
        for l, per in enumerate(S.lora_init(self.shape)):
            for name, t in per.items():
                for ab in ("A", "B"):
                    self.view(self.master, l, name, ab).copy_(t[ab])
        L.lsq_lora_refresh_bf16(self.master, self.op, self.numel)

    def init_device(self, seed: int = S.LORA_SEED):
        for l in range(self.shape.n_layers):
            for i, (name, (n, k)) in enumerate(self.shape.linear_shapes().items()):
                st = 1000 + 16 * l + i
                self.view(self.master, l, name, "A").copy_(
                    S.device_normal_f32((self.shape.r, k), 1.0 / math.sqrt(k), seed, st))
                self.view(self.master, l, name, "B").copy_(
                    S.device_normal_f32((n, self.shape.r), S.LORA_B_STD, seed, st + 8))
        L.lsq_lora_refresh_bf16(self.master, self.op, self.numel)


@dataclasses.dataclass
class _StepGraph:
    """One recorded forward/backward: the graph, the kernels it launches, the scheduler counters
    (uploads, bytes, reused per scheduler) one step advances, and whether it has run."""
    graph: "torch.cuda.CUDAGraph"
    launches: int
    stats_delta: list
    ran: bool = False

    def replay(self):
        self.graph.replay()


class StreamedLoraTrainer:
    """One GPU, one batch of [batch, seq] token ids per step.

    n_slots: HBM slots for streamed layer records (2..8), or None for a
    resident run (one slot per layer, every layer uploaded once).
    init: "host" draws every weight from the seeded numpy streams that the
    oracle also reads; "device" draws them with the CUDA RNG (full-size runs).
    head: "hbm" keeps the lm_head resident; "host" keeps it in page-locked
    host RAM and streams it in vocabulary chunks of head_chunk rows through
    two HBM chunk buffers on the copy stream, once for each of its GEMMs (with
    a tied embedding the one host table also serves the gather, zero-copy).
    The chunked GEMMs give bit for bit the resident head's results.
    """

    def __init__(self, shape: S.ModelShape, batch: int, seq: int, n_slots: Optional[int] = 2,
                 init: str = "device", lr: float = 2e-5, device: str = "cuda", share: "StreamedLoraTrainer" = None,
                 absmax: str = "fp32", shard: Optional[tuple] = None, source: str = "ram",
                 store_path: Optional[str] = None, embed: str = "hbm", head: str = "hbm",
                 head_chunk: int = 8192, graph: bool = False):
        self.shape, self.B, self.S = shape, batch, seq
        self.timeline = None   # list of (kind, flops, start_event, end_event) when instrumented
        self.M = batch * seq
        self.lr = lr
        self.dev = device
        self.resident = n_slots is None
        self.n_slots = shape.n_layers if self.resident else int(n_slots)
        # shard = (rank, world): sharded upload over the default process group (each rank
        # pins and copies 1/world of every record; an all-gather completes the slot)
        self.shard = None if shard is None else (int(shard[0]), int(shard[1]))
        align = 4096 if self.shard is None else math.lcm(4096, 256 * self.shard[1])
        self.layout = RecordLayout.of(shape, absmax, align)
        self.absmax_kind = absmax
        # source "disk": the records live in a file (store_path) and reach the GPU through
        # page-locked staging buffers filled by the library's reader threads
        if source not in ("ram", "disk") or (source == "disk") != (store_path is not None):
            raise ValueError("source must be 'ram', or 'disk' with a store_path")
        self.source, self.store_path = source, store_path
        # embed "host": an untied embedding table stays in page-locked host RAM and the
        # gather reads the batch's rows straight over the host link (zero-copy)
        if embed not in ("hbm", "host") or (embed == "host" and shape.tied):
            raise ValueError("embed must be 'hbm', or 'host' for an untied embedding")
        self.embed_kind = embed
        if head not in ("hbm", "host") or head_chunk < 64 or head_chunk % 256 != 0:
            raise ValueError("head must be 'hbm' or 'host'; head_chunk a positive multiple of 256 rows")
        self.head_kind, self.head_chunk = head, int(head_chunk)
        if head == "host" and shape.tied:
            self.embed_kind = embed = "host"   # one table: the head's host copy also serves the gather
        self.compute = torch.cuda.current_stream()
        self.copy = torch.cuda.Stream()
        # graph: after a warm-up step, each kind of forward/backward is recorded once as a CUDA graph
        # (the step's kernels, uploads and events) and replayed, so its launches are read from device
        # memory instead of over the host link that the layer copies keep busy
        self.graph = bool(graph)
        if self.graph and (self.compute.cuda_stream == 0 or source == "disk" or shard is not None):
            raise ValueError("graph replay needs a non-default compute stream (construct and drive the trainer "
                             "under torch.cuda.stream(...)) and the host-RAM tier without sharding")
        self._graphs = {}       # kind -> _StepGraph
        self._stats_extra = [[0, 0, 0], [0, 0, 0]]   # counters of replays (layers, head)
        self._warm = set()      # kinds that ran eagerly since the last residency change
        if share is not None and (share.absmax_kind != absmax or share.shard != self.shard or
                                  (share.source, share.store_path, share.embed_kind, share.head_kind,
                                   share.head_chunk) != (source, store_path, embed, head, self.head_chunk)):
            raise ValueError("a shared store must have the same absmax format, sharding, source, embed and head "
                             "places")
        if share is not None:       # reuse another trainer's host store and resident tensors
            self.host_records = share.host_records
            self.embed, self.lm_head, self.final_norm = share.embed, share.lm_head, share.final_norm
        else:
            self._build_store(init)
            self._build_resident(init)
        self.lora = LoraParams(shape, device)
        if init == "host":
            self.lora.init_host()
        else:
            self.lora.init_device()
        self._alloc_activations()
        self.slots = [torch.empty(self.layout.slot_bytes, dtype=torch.uint8, device=device)
                      for _ in range(self.n_slots)]
        lo, hi = self.shard_range()
        disk = None
        if source == "disk":
            self.staging = [torch.empty(hi - lo, dtype=torch.uint8, pin_memory=True) for _ in range(3)]
            disk = (store_path, [b.data_ptr() for b in self.staging], 4)
        self.sched = L.lsq_stream_create(shape.n_layers, self.n_slots, self.layout.nbytes,
                                         [s.data_ptr() for s in self.slots],
                                         None if source == "disk" else [h.data_ptr() for h in self.host_records],
                                         self.compute, self.copy,
                                         shard=None if self.shard is None else (*self.shard, lambda *a: self._gather(*a)),
                                         disk=disk)
        if self.layout.dq:
            L.lsq_stream_set_absmax_expand(self.sched, self.layout.expand_items(), self.layout.slot_bytes)
        self.head_sched = None
        if self.head_kind == "host":
            # the head's chunks are the "layers" of a second scheduler: same copy stream, two slots
            C, d = self.head_chunk, shape.d
            self.head_chunks = -(-shape.vocab // C)
            cbytes = C * d * 2
            self.head_slots = [torch.empty(cbytes, dtype=torch.uint8, device=device) for _ in range(2)]
            base = self.lm_head.data_ptr()
            self.head_sched = L.lsq_stream_create(self.head_chunks, 2, cbytes, [t.data_ptr() for t in self.head_slots],
                                                  [base + c * cbytes for c in range(self.head_chunks)],
                                                  self.compute, self.copy)
            self.dh32 = torch.empty(self.M, d, dtype=torch.float32, device=device)
        if self.resident:
            for l in range(shape.n_layers):
                L.lsq_layer_upload_async(self.sched, l, l)
            torch.cuda.synchronize()
        self.loss_dev = torch.zeros(1, dtype=torch.float32, device=device)

    # ------------------------------------------------------------------ setup
    def shard_range(self):
        """Bytes of every record this rank pins and copies: [lo, hi)."""
        if self.shard is None:
            return 0, self.layout.nbytes
        return DP.shard_range(self.layout.nbytes, *self.shard)

    def _gather(self, layer, slot, slot_ptr, nbytes, stream_handle):
        """Sharded upload: after this rank's part of the record landed in the slot
        (on the copy stream), complete the slot from the other ranks - an in-place
        all-gather over the default process group, ordered on the copy stream."""
        t = self.slots[slot]
        assert t.data_ptr() == slot_ptr and stream_handle == self.copy.cuda_stream and nbytes == self.layout.nbytes
        DP.gather_slot(t, nbytes, *self.shard, stream=self.copy)

    def _build_store(self, init: str):
        """Quantise every layer once on the GPU and keep the records pinned on the host
        (source "ram"), or write this rank's parts of them back to back to store_path
        (source "disk")."""
        sh, lay = self.shape, self.layout
        stage = torch.zeros(lay.slot_bytes, dtype=torch.uint8, device=self.dev)
        base = stage.data_ptr()
        self.host_records: List[torch.Tensor] = []
        fout = open(self.store_path, "wb") if self.source == "disk" else None
        for l in range(sh.n_layers):
            if init == "host":
                Wl = S.layer_weights(sh, l)
            for i, (name, (n, k)) in enumerate(sh.linear_shapes().items()):
                if init == "host":
                    w = Wl[name].to(self.dev)
                else:
                    w = S.device_normal_bf16((n, k), S.BASE_STD, S.WEIGHT_SEED, 1000 + 16 * l + i)
                L.lsq_nf4_quantize(w, base + lay.codes[name], base + lay.absmax[name])
                if lay.dq:   # second level: the record keeps the 8-bit codes and block params
                    c8, pp, nb = lay.dq[name]
                    L.lsq_absmax_double_quantize(base + lay.absmax[name], nb, base + c8, base + pp)
                del w
            ones = torch.ones(sh.d, dtype=torch.bfloat16, device=self.dev)
            stage[lay.ln1:lay.ln1 + 2 * sh.d].copy_(ones.view(torch.uint8))
            stage[lay.ln2:lay.ln2 + 2 * sh.d].copy_(ones.view(torch.uint8))
            lo, hi = self.shard_range()
            if fout is not None:
                fout.write(stage[lo:hi].cpu().numpy().tobytes())
                continue
            rec = torch.empty(hi - lo, dtype=torch.uint8, pin_memory=True)
            rec.copy_(stage[lo:hi])
            self.host_records.append(rec)
        if fout is not None:
            fout.close()
        del stage
        torch.cuda.synchronize()

    def _build_resident(self, init: str):
        sh = self.shape
        if init == "host":
            e = S.embeddings(sh)
            self.embed = e["embed"].to(self.dev)
            self.lm_head = self.embed if sh.tied else e["lm_head"].to(self.dev)
        else:
            self.embed = S.device_normal_bf16((sh.vocab, sh.d), S.BASE_STD, S.WEIGHT_SEED, 11)
            self.lm_head = self.embed if sh.tied else S.device_normal_bf16((sh.vocab, sh.d), S.BASE_STD,
                                                                            S.WEIGHT_SEED, 12)
        if self.head_kind == "host":
            # page-locked host copy, padded to whole chunks (every chunk upload copies the same bytes)
            rows = -(-sh.vocab // self.head_chunk) * self.head_chunk
            host = torch.zeros(rows, sh.d, dtype=self.lm_head.dtype, pin_memory=True)
            host[:sh.vocab].copy_(self.lm_head)
            if sh.tied:
                self.embed = host
            self.lm_head = host
        if self.embed_kind == "host" and not self.embed.is_pinned():   # the gather reads it in place
            host = torch.empty(self.embed.shape, dtype=self.embed.dtype, pin_memory=True)
            host.copy_(self.embed)
            self.embed = host
        self.final_norm = torch.ones(sh.d, dtype=torch.bfloat16, device=self.dev)

    def _alloc_activations(self):
        sh, M, dev = self.shape, self.M, self.dev
        bf = dict(dtype=torch.bfloat16, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        d, f, kv, r = sh.d, sh.f, sh.kv, sh.r
        self.ids = torch.zeros(M, dtype=torch.int32, device=dev)
        self.h = torch.empty(sh.n_layers + 1, M, d, **bf)        # checkpointed layer inputs
        self.x1, self.q, self.a, self.hmid, self.x2 = (torch.empty(M, d, **bf) for _ in range(5))
        self.k, self.v = torch.empty(M, kv, **bf), torch.empty(M, kv, **bf)
        self.g, self.u, self.mm = (torch.empty(M, f, **bf) for _ in range(3))
        self.rstd1, self.rstd2, self.rstdf = (torch.empty(M, **f32) for _ in range(3))
        self.lse = torch.empty(self.B * sh.n_q * self.S, **f32)
        self.U = {n: torch.empty(M, r, **f32) for n in S.LINEARS}
        # rank state of every fused linear of every layer: the first forward fills it, the
        # checkpoint recompute and the backward read it (no rank-r kernels in the recompute)
        self.keep_rank_state = True
        self._groups = {"qkv": ([d, kv, kv], d), "o": ([d], d), "gateup": ([f, f], d), "down": ([d], f)}
        sizes = {g: _al(L.lsq_nf4_lora_state_size(ns, M, k, r)) for g, (ns, k) in self._groups.items()}
        per_layer = sum(sizes.values())
        self.rank_state_buf = torch.empty(sh.n_layers * per_layer, dtype=torch.uint8, device=dev)
        self.rank_state = []
        for l in range(sh.n_layers):
            off, views = l * per_layer, {}
            for g, sz in sizes.items():
                views[g] = self.rank_state_buf[off:off + sz]
                off += sz
            self.rank_state.append(views)
        self.dh, self.dhmid, self.dx, self.dq, self.da = (torch.empty(M, d, **bf) for _ in range(5))
        self.dk, self.dv = torch.empty(M, kv, **bf), torch.empty(M, kv, **bf)
        self.dmm = torch.empty(M, f, **bf)
        self.hn = torch.empty(M, d, **bf)
        self.logits = torch.empty(M, sh.vocab, **f32)
        self.dlogits = torch.empty(M, sh.vocab, **bf)
        # one scratch buffer serves every fused linear, forward and backward (they run in order on one stream)
        groups = [([d, kv, kv], d), ([d], d), ([f, f], d), ([d], f)]
        ws = max(max(L.lsq_nf4_lora_bwd_workspace_size(ns, M, k, r), L.lsq_nf4_lora_fwd_workspace_size(ns, M, k, r))
                 for ns, k in groups)
        self.ws_lora = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(L.lsq_attention_bwd_workspace_size(self.B, self.S, sh.n_q), dtype=torch.uint8,
                                   device=dev)
        self.ws_xent = torch.empty(L.lsq_xent_workspace_size(M), dtype=torch.uint8, device=dev)
        # RoPE: (cos, sin) per position and frequency; with head dims the fused GEMM epilogue serves,
        # q and k are rotated there and the attention backward returns their unrotated gradients
        self.rope_table = L.rope_table(sh.theta, self.S, sh.hd, device=dev)
        self.fuse_rope = sh.hd in (64, 128, 256)

    # ------------------------------------------------------------------ timing
    def _t0(self):
        if self.timeline is None:
            return None
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.compute)
        return e

    def _t1(self, start, kind: str, flops: float):
        if start is None:
            return
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.compute)
        self.timeline.append((kind, flops, start, e))

    def _fwd_flops(self, ns, K, r_down=None, r_up=None):
        """FLOPs of one fused forward call: the base GEMM, U = X A^T when this call computes it
        (r_down), and the LoRA-up block (r_up)."""
        M = self.M
        r_down = self.shape.r if r_down is None else r_down
        r_up = r_down if r_up is None else r_up
        return sum(2.0 * M * n * K + 2.0 * M * r_down * K + 2.0 * M * n * r_up for n in ns)

    def _bwd_flops(self, ns, K):
        M, r = self.M, self.shape.r
        return sum(2.0 * M * n * K + 2.0 * M * n * r + 2.0 * M * r * K for n in ns)

    # ------------------------------------------------------------------ layer
    def _ops(self, l: int):
        lp = self.lora
        A = {n: lp.view(lp.op, l, n, "A") for n in S.LINEARS}
        B = {n: lp.view(lp.op, l, n, "B") for n in S.LINEARS}
        return A, B

    def _layer_fwd(self, l: int, W: LayerView, save: bool, hin=None, hout=None, adapter: bool = True):
        """Layer l: hin (default h[l]) -> hout (default h[l+1], may alias hin).
        adapter=False runs the frozen base alone (r = 0): the reference model
        of the preference loss."""
        sh, M = self.shape, self.M
        r, s = (sh.r, sh.s) if adapter else (0, 0.0)
        if adapter:
            A, B = self._ops(l)
        else:
            A = B = {n: None for n in S.LINEARS}
        hin = self.h[l] if hin is None else hin
        hout = self.h[l + 1] if hout is None else hout
        U = self.U if save and adapter else {n: None for n in S.LINEARS}
        state = adapter and self.keep_rank_state
        ready = save           # the recompute: the first forward of this step filled the rank state
        rf = 0 if (state and ready) else r   # rank-r FLOPs done in this call

        def fused(group, Ws, x, names, res, ys, rope=None):
            if rope is not None:
                L.lsq_nf4_lora_fwd_multi_ex2(Ws, x, M, [A[n] for n in names], [B[n] for n in names], r, s, res, ys,
                                             None if state else [U[n] for n in names],
                                             self.rank_state[l][group] if state else None, ready, rope,
                                             workspace=self.ws_lora)
            elif state:
                L.lsq_nf4_lora_fwd_multi_ex(Ws, x, M, [A[n] for n in names], [B[n] for n in names], r, s, res, ys,
                                            None, self.rank_state[l][group], ready, workspace=self.ws_lora)
            else:
                L.lsq_nf4_lora_fwd_multi(Ws, x, M, [A[n] for n in names], [B[n] for n in names], r, s, res, ys,
                                         [U[n] for n in names], workspace=self.ws_lora)

        L.lsq_rmsnorm_fwd(hin, W.ln1, self.x1, self.rstd1, M, sh.d, sh.eps)
        t = self._t0()
        rope = (self.rope_table, self.S, sh.hd, 0b011) if self.fuse_rope else None   # q and k
        fused("qkv", [W.W["q"], W.W["k"], W.W["v"]], self.x1, ["q", "k", "v"], None, [self.q, self.k, self.v], rope)
        self._t1(t, "nf4_fwd", self._fwd_flops([sh.d, sh.kv, sh.kv], sh.d, rf, r))
        if not self.fuse_rope:
            L.lsq_rope(self.q, self.B, self.S, sh.n_q, sh.hd, sh.theta, 0)
            L.lsq_rope(self.k, self.B, self.S, sh.n_kv, sh.hd, sh.theta, 0)
        L.lsq_attention_fwd(self.q, self.k, self.v, self.a, self.lse, self.B, self.S, sh.n_q, sh.n_kv, sh.hd)
        t = self._t0()
        fused("o", [W.W["o"]], self.a, ["o"], [hin], [self.hmid])
        self._t1(t, "nf4_fwd", self._fwd_flops([sh.d], sh.d, rf, r))
        L.lsq_rmsnorm_fwd(self.hmid, W.ln2, self.x2, self.rstd2, M, sh.d, sh.eps)
        t = self._t0()
        fused("gateup", [W.W["gate"], W.W["up"]], self.x2, ["gate", "up"], None, [self.g, self.u])
        self._t1(t, "nf4_fwd", self._fwd_flops([sh.f, sh.f], sh.d, rf, r))
        L.lsq_swiglu_fwd(self.g, self.u, self.mm, M * sh.f)
        t = self._t0()
        fused("down", [W.W["down"]], self.mm, ["down"], [self.hmid], [hout])
        self._t1(t, "nf4_fwd", self._fwd_flops([sh.d], sh.f, rf, r))

    def _layer_bwd(self, l: int, W: LayerView):
        """self.dh holds dLoss/dh[l+1] on entry and dLoss/dh[l] on exit."""
        sh, M, r, s = self.shape, self.M, self.shape.r, self.shape.s
        A, B = self._ops(l)
        lp = self.lora
        gA = {n: lp.view(lp.grad, l, n, "A") for n in S.LINEARS}
        gB = {n: lp.view(lp.grad, l, n, "B") for n in S.LINEARS}
        U = self.U

        def fused_bwd(group, Ws, x, dys, names, dx):
            if self.keep_rank_state:
                L.lsq_nf4_lora_bwd_multi_ex(Ws, x, dys, M, [A[n] for n in names], [B[n] for n in names], r, s, None,
                                            self.rank_state[l][group], dx, [gA[n] for n in names],
                                            [gB[n] for n in names], 0, self.ws_lora)
            else:
                L.lsq_nf4_lora_bwd_multi(Ws, x, dys, M, [A[n] for n in names], [B[n] for n in names], r, s,
                                         [U[n] for n in names], dx, [gA[n] for n in names], [gB[n] for n in names],
                                         0, self.ws_lora)

        # down:  h_out = h_mid + down(m)
        t = self._t0()
        fused_bwd("down", [W.W["down"]], self.mm, [self.dh], ["down"], self.dmm)
        self._t1(t, "nf4_bwd", self._bwd_flops([sh.d], sh.f))
        L.lsq_swiglu_bwd(self.dmm, self.g, self.u, self.g, self.u, M * sh.f)   # g, u <- dg, du
        t = self._t0()
        fused_bwd("gateup", [W.W["gate"], W.W["up"]], self.x2, [self.g, self.u], ["gate", "up"], self.dx)
        self._t1(t, "nf4_bwd", self._bwd_flops([sh.f, sh.f], sh.d))
        L.lsq_rmsnorm_bwd(self.dx, self.hmid, W.ln2, self.rstd2, self.dh, self.dhmid, M, sh.d)
        # o:  h_mid = h_in + o(a)
        t = self._t0()
        fused_bwd("o", [W.W["o"]], self.a, [self.dhmid], ["o"], self.da)
        self._t1(t, "nf4_bwd", self._bwd_flops([sh.d], sh.d))
        L.lsq_attention_bwd_ex(self.q, self.k, self.v, self.a, self.lse, self.da, self.dq, self.dk, self.dv, self.B,
                               self.S, sh.n_q, sh.n_kv, sh.hd, self.rope_table if self.fuse_rope else None,
                               self.ws_attn)
        if not self.fuse_rope:
            L.lsq_rope(self.dq, self.B, self.S, sh.n_q, sh.hd, sh.theta, 1)
            L.lsq_rope(self.dk, self.B, self.S, sh.n_kv, sh.hd, sh.theta, 1)
        t = self._t0()
        fused_bwd("qkv", [W.W["q"], W.W["k"], W.W["v"]], self.x1, [self.dq, self.dk, self.dv], ["q", "k", "v"],
                  self.dx)
        self._t1(t, "nf4_bwd", self._bwd_flops([sh.d, sh.kv, sh.kv], sh.d))
        L.lsq_rmsnorm_bwd(self.dx, self.h[l], W.ln1, self.rstd1, self.dhmid, self.dh, M, sh.d)

    def _head_chunk_rows(self, c: int):
        r0 = c * self.head_chunk
        return r0, min(self.head_chunk, self.shape.vocab - r0)

    def _head_logits(self):
        """logits = hn E^T (fp32): one GEMM over the resident head, or one per streamed chunk,
        each writing its block of logit columns."""
        sh, M = self.shape, self.M
        if self.head_sched is None:
            L.lsq_dense_gemm(self.hn, self.lm_head, self.logits, M, sh.vocab, sh.d, 0, 1)
            return
        for c in range(self.head_chunks):
            Ec = L.lsq_stream_step(self.head_sched, c, +1)
            r0, rows = self._head_chunk_rows(c)
            L.lsq_dense_gemm_ex(self.hn, sh.d, Ec, self.logits.data_ptr() + 4 * r0, sh.vocab, None, M, rows, sh.d,
                                0, 1)

    def _head_dh(self):
        """hn <- dlogits E: one GEMM over the resident head, or the contraction over the vocabulary
        split at the streamed chunks, each call continuing from the fp32 accumulator the previous
        left (bit-identical to the one GEMM)."""
        sh, M = self.shape, self.M
        if self.head_sched is None:
            L.lsq_dense_gemm(self.dlogits, self.lm_head, self.hn, M, sh.d, sh.vocab, 1, 0)
            return
        last = self.head_chunks - 1
        for c in range(self.head_chunks):
            Ec = L.lsq_stream_step(self.head_sched, c, +1)
            r0, rows = self._head_chunk_rows(c)
            L.lsq_dense_gemm_ex(self.dlogits.data_ptr() + 2 * r0, sh.vocab, Ec, self.hn if c == last else self.dh32,
                                sh.d, None if c == 0 else self.dh32, M, sh.d, rows, 1, 0 if c == last else 1)

    def _view(self, l: int, direction: int) -> LayerView:
        return LayerView(self.shape, self.layout, L.lsq_stream_step(self.sched, l, direction))

    # ------------------------------------------------------------------ step
    def set_ids(self, ids: torch.Tensor):
        self.ids.copy_(ids.reshape(-1).to(torch.int32), non_blocking=True)

    # ------------------------------------------------------------------ graph replay
    def _scheds(self):
        return [s for s in (self.sched, self.head_sched) if s is not None]

    def _raw_stats(self):
        return [L.lsq_stream_stats(s) for s in self._scheds()]

    def _graphed(self, kind, body):
        """Run one forward/backward of this kind: eagerly while warming up or instrumented, else by
        replaying its recorded graph (recorded at the first call after an eager warm-up step)."""
        if not self.graph or self.timeline is not None:
            body()
            self._warm.add(kind)
            return
        g = self._graphs.get(kind)
        if g is None:
            if kind not in self._warm:      # the first step of a walk fills the slots: not periodic yet
                body()
                self._warm.add(kind)
                return
            g = self._capture(kind, body)
        self.compute.wait_stream(self.copy)   # eager uploads queued before this step come first
        g.replay()
        if g.ran:                             # the capture advanced the counters once already
            L.LAUNCHES[0] += g.launches
            for k, d in enumerate(g.stats_delta):
                self._stats_extra[k] = [a + b for a, b in zip(self._stats_extra[k], d)]
        g.ran = True

    def _capture(self, kind, body):
        scheds = self._scheds()
        before, launches0 = self._raw_stats(), L.LAUNCHES[0]
        graph = torch.cuda.CUDAGraph()
        opened = []
        try:
            with torch.cuda.graph(graph, stream=self.compute, capture_error_mode="thread_local"):
                for sc in scheds:
                    L.lsq_stream_capture_begin(sc)
                    opened.append(sc)
                body()
                while opened:
                    L.lsq_stream_capture_end(opened.pop(0))
        except BaseException:
            for sc in opened:
                try:
                    L.lsq_stream_capture_end(sc)
                except L.LsqError:
                    pass
            # the policy advanced as if the captured step had run: forget residency so that the
            # next step uploads what it needs
            torch.cuda.synchronize()
            for sc in scheds:
                L.lsq_stream_reset(sc)
            self._warm.clear()
            raise
        after = self._raw_stats()
        g = _StepGraph(graph, L.LAUNCHES[0] - launches0,
                       [[a - b for a, b in zip(x, y)] for x, y in zip(after, before)])
        self._graphs[kind] = g
        return g

    def drop_graphs(self):
        """Forget the recorded steps (the next step of each kind runs eagerly and records again)."""
        torch.cuda.synchronize()
        self._graphs.clear()

    def forward_backward(self):
        """Loss into self.loss_dev and LoRA gradients into self.lora.grad."""
        self._graphed("sft", self._forward_backward)

    def _forward_backward(self):
        sh, M = self.shape, self.M
        L.lsq_embed_gather(self.ids, self.embed, self.h[0], M, sh.d, sh.vocab)
        for l in range(sh.n_layers):
            self._layer_fwd(l, self._view(l, +1), save=False)
        L.lsq_rmsnorm_fwd(self.h[sh.n_layers], self.final_norm, self.hn, self.rstdf, M, sh.d, sh.eps)
        self._head_logits()
        L.lsq_xent_fwd_bwd(self.logits, self.ids, self.B, self.S, sh.vocab, self.loss_dev, self.dlogits,
                           self.ws_xent)
        self._head_dh()   # hn <- d hn
        L.lsq_rmsnorm_bwd(self.hn, self.h[sh.n_layers], self.final_norm, self.rstdf, None, self.dh, M, sh.d)
        for l in reversed(range(sh.n_layers)):
            W = self._view(l, -1)
            self._layer_fwd(l, W, save=True)
            self._layer_bwd(l, W)

    def _dpo_buffers(self):
        if getattr(self, "h_ref", None) is None:
            dev, M = self.h.device, self.M
            self.h_ref = torch.empty(M, self.shape.d, dtype=torch.bfloat16, device=dev)
            self.row_lse = torch.empty(M, dtype=torch.float32, device=dev)
            self.pi_logp, self.ref_logp, self.dseq = (torch.empty(self.B, dtype=torch.float32, device=dev)
                                                      for _ in range(3))
            self.ws_seqlp = torch.empty(L.lsq_seq_logprob_workspace_size(M), dtype=torch.uint8, device=dev)

    def forward_backward_dpo(self, beta: float = 0.1):
        if self.B % 2:
            raise ValueError("DPO needs an even batch (pairs of chosen / rejected sequences)")
        self._dpo_buffers()
        self._graphed(("dpo", float(beta)), lambda: self._forward_backward_dpo(beta))

    def _forward_backward_dpo(self, beta: float = 0.1):
        """DPO over the batch as pairs (chosen = sequence 2i, rejected = 2i+1):
        loss into self.loss_dev, LoRA gradients into self.lora.grad.

        The reference model is the same streamed base with the adapters off:
        while a layer's record is on the GPU for the policy forward, the
        reference forward of that layer runs too (fused linears with r = 0), so
        the reference costs compute but no extra layer uploads."""
        sh, M = self.shape, self.M
        if self.B % 2:
            raise ValueError("DPO needs an even batch (pairs of chosen / rejected sequences)")
        self._dpo_buffers()
        L.lsq_embed_gather(self.ids, self.embed, self.h[0], M, sh.d, sh.vocab)
        L.lsq_embed_gather(self.ids, self.embed, self.h_ref, M, sh.d, sh.vocab)
        for l in range(sh.n_layers):
            W = self._view(l, +1)
            self._layer_fwd(l, W, save=False)
            self._layer_fwd(l, W, save=False, hin=self.h_ref, hout=self.h_ref, adapter=False)
        # reference sequence log-probabilities
        L.lsq_rmsnorm_fwd(self.h_ref, self.final_norm, self.hn, self.rstdf, M, sh.d, sh.eps)
        self._head_logits()
        L.lsq_seq_logprob(self.logits, self.ids, self.B, self.S, sh.vocab, self.row_lse, self.ref_logp, self.ws_seqlp)
        # policy sequence log-probabilities, loss, d loss / d logits
        L.lsq_rmsnorm_fwd(self.h[sh.n_layers], self.final_norm, self.hn, self.rstdf, M, sh.d, sh.eps)
        self._head_logits()
        L.lsq_seq_logprob(self.logits, self.ids, self.B, self.S, sh.vocab, self.row_lse, self.pi_logp, self.ws_seqlp)
        L.lsq_dpo_loss(self.pi_logp, self.ref_logp, self.B // 2, beta, self.loss_dev, self.dseq)
        L.lsq_seq_logprob_bwd(self.logits, self.ids, self.B, self.S, sh.vocab, self.row_lse, self.dseq,
                              self.dlogits)
        self._head_dh()   # hn <- d hn
        L.lsq_rmsnorm_bwd(self.hn, self.h[sh.n_layers], self.final_norm, self.rstdf, None, self.dh, M, sh.d)
        for l in reversed(range(sh.n_layers)):
            W = self._view(l, -1)
            self._layer_fwd(l, W, save=True)
            self._layer_bwd(l, W)

    def train_step_dpo(self, ids: Optional[torch.Tensor] = None, beta: float = 0.1):
        if ids is not None:
            self.set_ids(ids)
        self.forward_backward_dpo(beta)
        self.optimizer_step()

    def optimizer_step(self):
        lp = self.lora
        lp.step += 1
        L.lsq_adamw_step(lp.master, lp.grad, lp.m, lp.v, lp.op, lp.numel, lp.step, self.lr, 0.9, 0.999, 1e-8, 0.0)

    def train_step(self, ids: Optional[torch.Tensor] = None):
        if ids is not None:
            self.set_ids(ids)
        self.forward_backward()
        self.optimizer_step()

    def logits_of_last_forward(self) -> torch.Tensor:
        return self.logits

    def stats(self):
        """(uploads, bytes, reused) of the layer records since create, replayed steps included."""
        return tuple(a + b for a, b in zip(L.lsq_stream_stats(self.sched), self._stats_extra[0]))

    def head_stats(self):
        """(uploads, bytes, reused) of the streamed head's chunks; zeros with a resident head."""
        if self.head_sched is None:
            return (0, 0, 0)
        return tuple(a + b for a, b in zip(L.lsq_stream_stats(self.head_sched), self._stats_extra[1]))

    def check_device(self):
        """Raise LsqError if a bounded wait inside any kernel ran out since the
        last check (the library's device status word, which the read clears):
        a kernel that gave up leaves its outputs incomplete, so no loss,
        gradient or timing of those steps stands.  Synchronises the device."""
        torch.cuda.synchronize()
        status, where = L.lsq_device_status()
        if status != 0:
            self._graphs.clear()   # a recorded step is not replayed after a kernel gave up
            raise L.LsqError(status, "device status word",
                             f"a bounded device wait gave up (site {where}); results since the last check are void")

    def close(self):
        if getattr(self, "_graphs", None):
            torch.cuda.synchronize()
            self._graphs.clear()
        if getattr(self, "head_sched", None):
            torch.cuda.synchronize()
            L.lsq_stream_destroy(self.head_sched)
            self.head_sched = None
        if getattr(self, "sched", None):
            torch.cuda.synchronize()
            L.lsq_stream_destroy(self.sched)
            self.sched = None
            self.check_device()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
