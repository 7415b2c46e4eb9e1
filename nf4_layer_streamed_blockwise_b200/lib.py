"""ctypes binding of the lsq C ABI (include/lsq.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (or raw ints for pointers) and passes their device addresses, sizes
and the stream handle through.  No computation happens on this side.  The
shared library is loaded from this package directory; if it is missing the
import fails loudly (there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsq.so")

c_void_p = ctypes.c_void_p
c_int32 = ctypes.c_int32
c_int64 = ctypes.c_int64
c_float = ctypes.c_float
c_size_t = ctypes.c_size_t

STATUS = {0: "LSQ_OK", 1: "LSQ_EINVAL", 2: "LSQ_ENOTPINNED", 3: "LSQ_ECUDA", 4: "LSQ_ETIMEOUT",
          5: "LSQ_ESTATE", 6: "LSQ_EUNSUPPORTED", 7: "LSQ_ECALLBACK"}


class LsqError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {msg}")
        self.status = status


class lsq_nf4_weight(ctypes.Structure):
    _fields_ = [("codes", c_void_p), ("absmax", c_void_p), ("n_out", c_int64), ("k_in", c_int64)]


class lsq_rope_spec(ctypes.Structure):
    _fields_ = [("table", c_void_p), ("seq", c_int32), ("hd", c_int32), ("segments", c_int32)]


class lsq_absmax_dq_item(ctypes.Structure):
    _fields_ = [("codes_off", ctypes.c_uint64), ("params_off", ctypes.c_uint64), ("out_off", ctypes.c_uint64),
                ("nb", c_int64)]


# int32 gather(void* user, int32 layer, int32 slot, void* slot_ptr, size_t record_bytes, cudaStream_t copy)
lsq_gather_fn = ctypes.CFUNCTYPE(c_int32, c_void_p, c_int32, c_int32, c_void_p, c_size_t, c_void_p)


class lsq_stream_cfg(ctypes.Structure):
    _fields_ = [("n_layers", c_int32), ("n_slots", c_int32), ("record_bytes", c_size_t),
                ("slots", ctypes.POINTER(c_void_p)), ("host_records", ctypes.POINTER(c_void_p)),
                ("shard_rank", c_int32), ("shard_world", c_int32), ("gather", lsq_gather_fn),
                ("gather_user", c_void_p), ("disk_path", ctypes.c_char_p), ("staging", ctypes.POINTER(c_void_p)),
                ("n_staging", c_int32), ("disk_threads", c_int32)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing; build it with `python -m nf4_layer_streamed_blockwise_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

_SIGS = {
    "lsq_status_str": (ctypes.c_char_p, [c_int32]),
    "lsq_last_error": (ctypes.c_char_p, []),
    "lsq_version": (c_int32, []),
    "lsq_device_status": (c_int32, [ctypes.POINTER(c_int32), ctypes.POINTER(c_int32)]),
    "lsq_wait_flag": (c_int32, [c_void_p, ctypes.c_uint64, c_int64, c_void_p]),
    "lsq_nf4_codebook": (c_int32, [ctypes.POINTER(c_float)]),
    "lsq_nf4_quantize": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_void_p]),
    "lsq_nf4_dequantize": (c_int32, [ctypes.POINTER(lsq_nf4_weight), c_void_p, c_void_p]),
    "lsq_absmax_double_quantize": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_void_p]),
    "lsq_absmax_expand": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p, c_void_p]),
    "lsq_nf4_lora_fwd_workspace_size": (c_size_t, [c_int32, c_int64, c_int64, ctypes.POINTER(c_int64), c_int32]),
    "lsq_nf4_lora_fwd": (c_int32, [ctypes.POINTER(lsq_nf4_weight), c_void_p, c_int64, c_void_p, c_void_p, c_int32,
                                   c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "lsq_nf4_lora_state_size": (c_size_t, [c_int32, c_int64, c_int64, ctypes.POINTER(c_int64), c_int32]),
    "lsq_nf4_lora_fwd_multi_ex": (c_int32, [c_int32, ctypes.POINTER(lsq_nf4_weight), c_void_p, c_int64,
                                            c_void_p, c_void_p, c_int32, c_float, c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_int32, c_void_p, c_size_t, c_void_p]),
    "lsq_nf4_lora_fwd_multi_ex2": (c_int32, [c_int32, ctypes.POINTER(lsq_nf4_weight), c_void_p, c_int64,
                                             c_void_p, c_void_p, c_int32, c_float, c_void_p, c_void_p, c_void_p,
                                             c_void_p, c_int32, ctypes.POINTER(lsq_rope_spec), c_void_p, c_size_t,
                                             c_void_p]),
    "lsq_rope_table": (c_int32, [c_float, c_int64, c_int64, c_void_p, c_void_p]),
    "lsq_rope_table_size": (c_size_t, [c_int64, c_int64]),
    "lsq_attention_bwd_ex": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int64, c_int64, c_void_p,
                                       c_void_p, c_size_t, c_void_p]),
    "lsq_nf4_lora_bwd_multi_ex": (c_int32, [c_int32, ctypes.POINTER(lsq_nf4_weight), c_void_p, c_void_p, c_int64,
                                            c_void_p, c_void_p, c_int32, c_float, c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_int32, c_void_p, c_size_t, c_void_p]),
    "lsq_nf4_lora_fwd_multi": (c_int32, [c_int32, ctypes.POINTER(lsq_nf4_weight), c_void_p, c_int64,
                                         ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p), c_int32, c_float,
                                         ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p),
                                         ctypes.POINTER(c_void_p), c_void_p, c_size_t, c_void_p]),
    "lsq_nf4_lora_bwd_workspace_size": (c_size_t, [c_int32, c_int64, c_int64, ctypes.POINTER(c_int64), c_int32]),
    "lsq_nf4_lora_bwd": (c_int32, [ctypes.POINTER(lsq_nf4_weight), c_void_p, c_void_p, c_int64, c_void_p, c_void_p,
                                   c_int32, c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_int32, c_void_p,
                                   c_size_t, c_void_p]),
    "lsq_nf4_lora_bwd_multi": (c_int32, [c_int32, ctypes.POINTER(lsq_nf4_weight), c_void_p,
                                         ctypes.POINTER(c_void_p), c_int64, ctypes.POINTER(c_void_p),
                                         ctypes.POINTER(c_void_p), c_int32, c_float, ctypes.POINTER(c_void_p),
                                         c_void_p, ctypes.POINTER(c_void_p), ctypes.POINTER(c_void_p), c_int32,
                                         c_void_p, c_size_t, c_void_p]),
    "lsq_nf4_lora_bwd_noalloc_max_scratch": (c_size_t, []),
    "lsq_nf4_lora_bwd_noalloc": (c_int32, [ctypes.POINTER(lsq_nf4_weight), c_void_p, c_void_p, c_int64, c_void_p,
                                           c_void_p, c_int32, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                                           c_int32, c_void_p]),
    "lsq_dense_gemm": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, c_int32, c_int32,
                                 c_void_p]),
    "lsq_dense_gemm_ex": (c_int32, [c_void_p, c_int64, c_void_p, c_void_p, c_int64, c_void_p, c_int64, c_int64,
                                    c_int64, c_int32, c_int32, c_void_p]),
    "lsq_rmsnorm_fwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_float, c_void_p]),
    "lsq_rmsnorm_bwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64,
                                  c_void_p]),
    "lsq_rope": (c_int32, [c_void_p, c_int64, c_int64, c_int64, c_int64, c_float, c_int32, c_void_p]),
    "lsq_attention_fwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64,
                                    c_int64, c_int64, c_void_p]),
    "lsq_attention_bwd_workspace_size": (c_size_t, [c_int64, c_int64, c_int64]),
    "lsq_attention_bwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_int64, c_int64, c_int64, c_int64, c_int64, c_void_p, c_size_t,
                                    c_void_p]),
    "lsq_swiglu_fwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_void_p]),
    "lsq_swiglu_bwd": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_void_p]),
    "lsq_embed_gather": (c_int32, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int64, c_void_p]),
    "lsq_xent_workspace_size": (c_size_t, [c_int64]),
    "lsq_xent_fwd_bwd": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                   c_size_t, c_void_p]),
    "lsq_seq_logprob_workspace_size": (c_size_t, [c_int64]),
    "lsq_seq_logprob": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                  c_size_t, c_void_p]),
    "lsq_dpo_loss": (c_int32, [c_void_p, c_void_p, c_int32, c_float, c_void_p, c_void_p, c_void_p]),
    "lsq_seq_logprob_bwd": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p, c_void_p,
                                      c_void_p]),
    "lsq_lora_refresh_bf16": (c_int32, [c_void_p, c_void_p, c_int64, c_void_p]),
    "lsq_adamw_step": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int32, c_float,
                                 c_float, c_float, c_float, c_float, c_void_p]),
    "lsq_stream_create": (c_int32, [ctypes.POINTER(lsq_stream_cfg), c_void_p, c_void_p, ctypes.POINTER(c_void_p)]),
    "lsq_stream_set_absmax_expand": (c_int32, [c_void_p, ctypes.POINTER(lsq_absmax_dq_item), c_int32, c_size_t]),
    "lsq_layer_upload_async": (c_int32, [c_void_p, c_int32, c_int32]),
    "lsq_stream_step": (c_int32, [c_void_p, c_int32, c_int32, ctypes.POINTER(c_void_p)]),
    "lsq_stream_simulate": (c_int32, [c_int32, c_int32, c_int32, ctypes.POINTER(c_int32), ctypes.POINTER(c_int32),
                                      ctypes.POINTER(c_int32), c_int32, ctypes.POINTER(c_int32)]),
    "lsq_stream_stats": (c_int32, [c_void_p, ctypes.POINTER(c_int64), ctypes.POINTER(c_int64),
                                   ctypes.POINTER(c_int64)]),
    "lsq_stream_upload_ms": (c_int32, [c_void_p, c_int32, ctypes.POINTER(c_float)]),
    "lsq_stream_time_waits": (c_int32, [c_void_p, c_int32]),
    "lsq_stream_wait_ms": (c_int32, [c_void_p, ctypes.POINTER(c_float), ctypes.POINTER(c_float),
                                     ctypes.POINTER(c_int32), ctypes.POINTER(c_int32)]),
    "lsq_stream_reset": (c_int32, [c_void_p]),
    "lsq_stream_capture_begin": (c_int32, [c_void_p]),
    "lsq_stream_capture_end": (c_int32, [c_void_p]),
    "lsq_stream_destroy": (c_int32, [c_void_p]),
}


def _fn(name):
    f = getattr(_lib, name)
    res, args = _SIGS[name]
    f.restype, f.argtypes = res, args
    return f


def exported_symbols() -> list:
    """Names of the declared entry points that the loaded library exports."""
    out = []
    for name in _SIGS:
        try:
            getattr(_lib, name)
            out.append(name)
        except AttributeError:
            pass
    return out


def _check(name: str, status: int):
    if status != 0:
        msg = _fn("lsq_last_error")().decode(errors="replace")
        raise LsqError(status, name, msg)


# kernel launches issued by the library, counted per call on this side
# (with a LoRA adapter the fused linear's forward is 2 kernels: the rank-r
# product U = X A^T and the main GEMM, plus the operand transposition when a
# rank state is filled, and only the main GEMM when the state is reused; the
# backward is the operand padding (not with a state), G = dY B, the dX GEMM
# when dx is wanted, and the dA/dB GEMM with its reduction)
LAUNCHES = [0]
_KERNELS = {"lsq_nf4_quantize": 1, "lsq_nf4_dequantize": 1, "lsq_absmax_double_quantize": 1, "lsq_absmax_expand": 1,
            "lsq_dense_gemm": 1, "lsq_dense_gemm_ex": 1, "lsq_rmsnorm_fwd": 1, "lsq_rmsnorm_bwd": 1, "lsq_rope": 1, "lsq_rope_table": 1,
            "lsq_attention_fwd": 1, "lsq_attention_bwd": 3, "lsq_swiglu_fwd": 1, "lsq_swiglu_bwd": 1,
            "lsq_embed_gather": 1, "lsq_xent_fwd_bwd": 2, "lsq_adamw_step": 1, "lsq_lora_refresh_bf16": 1, "lsq_seq_logprob": 2,
            "lsq_dpo_loss": 1, "lsq_seq_logprob_bwd": 1, "lsq_wait_flag": 1}


def _call(name, *args, launches=None):
    _check(name, _fn(name)(*args))
    LAUNCHES[0] += _KERNELS.get(name, 0) if launches is None else launches


def _p(t) -> Optional[int]:
    """device / host address of a tensor (None for None; ints pass through)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptrs(seq) -> Optional[ctypes.Array]:
    if seq is None:
        return None
    arr = (c_void_p * len(seq))()
    for i, t in enumerate(seq):
        arr[i] = _p(t)
    return arr


class NF4Weight:
    """Device views of one NF4 weight: codes uint8 [n_out*k_in/2], absmax fp32 [n_out*k_in/64]."""

    def __init__(self, codes: torch.Tensor, absmax: torch.Tensor, n_out: int, k_in: int):
        self.codes, self.absmax, self.n_out, self.k_in = codes, absmax, int(n_out), int(k_in)

    def c(self) -> lsq_nf4_weight:
        return lsq_nf4_weight(_p(self.codes), _p(self.absmax), self.n_out, self.k_in)

    @staticmethod
    def empty(n_out: int, k_in: int, device="cuda") -> "NF4Weight":
        return NF4Weight(torch.empty(n_out * k_in // 2, dtype=torch.uint8, device=device),
                         torch.empty(n_out * (k_in // 64), dtype=torch.float32, device=device), n_out, k_in)


# ---------------------------------------------------------------------------- misc
def lsq_status_str(s: int) -> str:
    return _fn("lsq_status_str")(s).decode()


def lsq_last_error() -> str:
    return _fn("lsq_last_error")().decode(errors="replace")


def lsq_version() -> int:
    return _fn("lsq_version")()


def lsq_device_status():
    s, w = c_int32(0), c_int32(0)
    _call("lsq_device_status", ctypes.byref(s), ctypes.byref(w))
    return s.value, w.value


def lsq_wait_flag(flag, value: int, limit_ns: int, stream=None):
    """Stream-ordered wait until the 8-byte device word `flag` equals `value`; after limit_ns
    the wait gives up and the device status word reads (LSQ_ETIMEOUT, 901)."""
    _call("lsq_wait_flag", _p(flag), value, limit_ns, _stream(stream))


def lsq_nf4_codebook():
    out = (c_float * 16)()
    _call("lsq_nf4_codebook", out)
    return list(out)


# ---------------------------------------------------------------------------- NF4
def lsq_nf4_quantize(w_bf16: torch.Tensor, codes: torch.Tensor, absmax: torch.Tensor, stream=None):
    n, k = w_bf16.shape
    _call("lsq_nf4_quantize", _p(w_bf16), n, k, _p(codes), _p(absmax), _stream(stream))


def lsq_nf4_dequantize(w: NF4Weight, out_bf16: torch.Tensor, stream=None):
    cw = w.c()
    _call("lsq_nf4_dequantize", ctypes.byref(cw), _p(out_bf16), _stream(stream))


def lsq_absmax_double_quantize(absmax, nb: int, codes, params, stream=None):
    """absmax fp32 [nb] -> codes u8 [nb], params fp32 [ceil(nb/256), 2] (centre, scale); device memory."""
    _call("lsq_absmax_double_quantize", _p(absmax), nb, _p(codes), _p(params), _stream(stream))


def lsq_absmax_expand(codes, params, nb: int, absmax, stream=None):
    _call("lsq_absmax_expand", _p(codes), _p(params), nb, _p(absmax), _stream(stream))


def lsq_nf4_lora_fwd_workspace_size(n_outs: Sequence[int], M: int, k_in: int, r: int) -> int:
    arr = (c_int64 * len(n_outs))(*n_outs)
    return int(_fn("lsq_nf4_lora_fwd_workspace_size")(len(n_outs), M, k_in, arr, r))


def _fwd_workspace(workspace, n_outs, M, k_in, r, device):
    """The caller's workspace, or (when None and r > 0) a fresh one of the size the library asks for."""
    if workspace is not None or r == 0:
        return workspace
    return torch.empty(lsq_nf4_lora_fwd_workspace_size(n_outs, M, k_in, r), dtype=torch.uint8, device=device)


def _nbytes(t) -> int:
    return t.numel() * t.element_size() if t is not None else 0


def lsq_nf4_lora_fwd(W: NF4Weight, x, M: int, A, B, r: int, s: float, residual, y, u_out, stream=None,
                     workspace=None):
    cw = W.c()
    ws = _fwd_workspace(workspace, [W.n_out], M, W.k_in, r, y.device)
    _call("lsq_nf4_lora_fwd", ctypes.byref(cw), _p(x), M, _p(A), _p(B), r, s, _p(residual), _p(y), _p(u_out),
          _p(ws), _nbytes(ws), _stream(stream), launches=2 if r > 0 else 1)


def lsq_nf4_lora_fwd_multi(Ws: Sequence[NF4Weight], x, M: int, A, B, r: int, s: float, residual, y, u_out,
                           stream=None, workspace=None):
    n = len(Ws)
    cws = (lsq_nf4_weight * n)(*[w.c() for w in Ws])
    res = residual if residual is not None else [None] * n
    uo = u_out if u_out is not None else [None] * n
    ws = _fwd_workspace(workspace, [w.n_out for w in Ws], M, Ws[0].k_in, r, y[0].device)
    _call("lsq_nf4_lora_fwd_multi", n, cws, _p(x), M, _ptrs(A), _ptrs(B), r, s, _ptrs(res), _ptrs(y), _ptrs(uo),
          _p(ws), _nbytes(ws), _stream(stream), launches=2 if r > 0 else 1)


def lsq_nf4_lora_bwd_workspace_size(n_outs: Sequence[int], M: int, k_in: int, r: int) -> int:
    arr = (c_int64 * len(n_outs))(*n_outs)
    return int(_fn("lsq_nf4_lora_bwd_workspace_size")(len(n_outs), M, k_in, arr, r))


def lsq_nf4_lora_bwd(W: NF4Weight, x, dy, M: int, A, B, r: int, s: float, u, dx, dA, dB, accumulate: int,
                     workspace, stream=None):
    cw = W.c()
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _call("lsq_nf4_lora_bwd", ctypes.byref(cw), _p(x), _p(dy), M, _p(A), _p(B), r, s, _p(u), _p(dx), _p(dA),
          _p(dB), accumulate, _p(workspace), wsb, _stream(stream), launches=_bwd_launches(r, dx))


def _bwd_launches(r: int, dx, state=None) -> int:
    return (1 if dx is not None else 0) + ((3 if state is not None else 4) if r > 0 else 0)


def lsq_nf4_lora_state_size(n_outs: Sequence[int], M: int, k_in: int, r: int) -> int:
    arr = (c_int64 * len(n_outs))(*n_outs)
    return int(_fn("lsq_nf4_lora_state_size")(len(n_outs), M, k_in, arr, r))


def lsq_nf4_lora_fwd_multi_ex(Ws: Sequence[NF4Weight], x, M: int, A, B, r: int, s: float, residual, y, u_out,
                              state, state_ready: bool, workspace=None, stream=None):
    """The fused forward with a rank state (see include/lsq.h): state_ready=False computes
    the rank-r side into state (and U into u_out), True reuses it (the recompute)."""
    n = len(Ws)
    cws = (lsq_nf4_weight * n)(*[w.c() for w in Ws])
    res = residual if residual is not None else [None] * n
    uo = u_out if u_out is not None else [None] * n
    launches = 1 if (r == 0 or state_ready) else 3
    _call("lsq_nf4_lora_fwd_multi_ex", n, cws, _p(x), M, _ptrs(A), _ptrs(B), r, s, _ptrs(res), _ptrs(y), _ptrs(uo),
          _p(state), 1 if state_ready else 0, _p(workspace), _nbytes(workspace), _stream(stream), launches=launches)


def lsq_nf4_lora_fwd_multi_ex2(Ws: Sequence[NF4Weight], x, M: int, A, B, r: int, s: float, residual, y, u_out,
                               state, state_ready: bool, rope, workspace=None, stream=None):
    """lsq_nf4_lora_fwd_multi_ex with RoPE in the epilogue: rope = (table, seq, hd, segment bits) or None;
    state None = the workspace form (lsq_nf4_lora_fwd_multi)."""
    n = len(Ws)
    cws = (lsq_nf4_weight * n)(*[w.c() for w in Ws])
    res = residual if residual is not None else [None] * n
    uo = u_out if u_out is not None else [None] * n
    spec = None
    if rope is not None:
        spec = lsq_rope_spec(_p(rope[0]), int(rope[1]), int(rope[2]), int(rope[3]))
    if state is None:
        workspace = _fwd_workspace(workspace, [w.n_out for w in Ws], M, Ws[0].k_in, r, y[0].device)
        launches = 2 if r > 0 else 1
    else:
        launches = 1 if (r == 0 or state_ready) else 3
    _call("lsq_nf4_lora_fwd_multi_ex2", n, cws, _p(x), M, _ptrs(A), _ptrs(B), r, s, _ptrs(res), _ptrs(y),
          _ptrs(uo), _p(state), 1 if state_ready else 0, None if spec is None else ctypes.byref(spec),
          _p(workspace), _nbytes(workspace), _stream(stream), launches=launches)


def lsq_rope_table_size(seq: int, hd: int) -> int:
    return _fn("lsq_rope_table_size")(seq, hd)


def lsq_rope_table(theta: float, seq: int, hd: int, table, stream=None):
    """(cos, sin) fp32 pairs [seq][hd/2] of the RoPE angles, then the hd/2 frequencies, into
    table (device, lsq_rope_table_size bytes)."""
    _call("lsq_rope_table", theta, seq, hd, _p(table), _stream(stream))


def rope_table(theta: float, seq: int, hd: int, device="cuda"):
    """A device buffer of lsq_rope_table_size bytes filled by lsq_rope_table (fp32 view)."""
    t = torch.empty(lsq_rope_table_size(seq, hd) // 4, dtype=torch.float32, device=device)
    lsq_rope_table(theta, seq, hd, t)
    return t


def lsq_nf4_lora_bwd_multi_ex(Ws: Sequence[NF4Weight], x, dy, M: int, A, B, r: int, s: float, u, state, dx, dA, dB,
                              accumulate: int, workspace, stream=None):
    n = len(Ws)
    cws = (lsq_nf4_weight * n)(*[w.c() for w in Ws])
    wsb = _nbytes(workspace)
    _call("lsq_nf4_lora_bwd_multi_ex", n, cws, _p(x), _ptrs(dy), M, _ptrs(A), _ptrs(B), r, s, _ptrs(u), _p(state),
          _p(dx), _ptrs(dA), _ptrs(dB), accumulate, _p(workspace), wsb, _stream(stream),
          launches=_bwd_launches(r, dx, state))


def lsq_nf4_lora_bwd_multi(Ws: Sequence[NF4Weight], x, dy, M: int, A, B, r: int, s: float, u, dx, dA, dB,
                           accumulate: int, workspace, stream=None):
    n = len(Ws)
    cws = (lsq_nf4_weight * n)(*[w.c() for w in Ws])
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _call("lsq_nf4_lora_bwd_multi", n, cws, _p(x), _ptrs(dy), M, _ptrs(A), _ptrs(B), r, s, _ptrs(u), _p(dx),
          _ptrs(dA), _ptrs(dB), accumulate, _p(workspace), wsb, _stream(stream), launches=_bwd_launches(r, dx))


def lsq_nf4_lora_bwd_noalloc_max_scratch() -> int:
    return int(_fn("lsq_nf4_lora_bwd_noalloc_max_scratch")())


def lsq_nf4_lora_bwd_noalloc(W: NF4Weight, x, dy, M: int, A, B, r: int, s: float, u, dx, dA, dB, accumulate: int,
                             stream=None):
    """lsq_nf4_lora_bwd without a workspace argument: the library's own fixed
    scratch array is used, for callers that cannot allocate device memory."""
    cw = W.c()
    _call("lsq_nf4_lora_bwd_noalloc", ctypes.byref(cw), _p(x), _p(dy), M, _p(A), _p(B), r, s, _p(u), _p(dx), _p(dA),
          _p(dB), accumulate, _stream(stream), launches=_bwd_launches(r, dx))


def lsq_dense_gemm(a, b, out, M: int, N: int, K: int, trans_b: int, out_f32: int, stream=None):
    _call("lsq_dense_gemm", _p(a), _p(b), _p(out), M, N, K, trans_b, out_f32, _stream(stream))


# ---------------------------------------------------------------------------- layer ops
def lsq_dense_gemm_ex(a, lda: int, b, out, ldo: int, acc_in, M: int, N: int, K: int, trans_b: int, out_f32: int,
                      stream=None):
    """a, b, out, acc_in: tensors or raw device addresses (column blocks pass as addresses)."""
    _call("lsq_dense_gemm_ex", _p(a), lda, _p(b), _p(out), ldo, _p(acc_in), M, N, K, trans_b, out_f32,
          _stream(stream))


def lsq_rmsnorm_fwd(x, g, y, rstd, rows: int, d: int, eps: float, stream=None):
    _call("lsq_rmsnorm_fwd", _p(x), _p(g), _p(y), _p(rstd), rows, d, eps, _stream(stream))


def lsq_rmsnorm_bwd(dy, x, g, rstd, dres_in, dres_out, rows: int, d: int, stream=None):
    _call("lsq_rmsnorm_bwd", _p(dy), _p(x), _p(g), _p(rstd), _p(dres_in), _p(dres_out), rows, d, _stream(stream))


def lsq_rope(x, batch: int, seq: int, heads: int, hd: int, theta: float, inverse: int, stream=None):
    _call("lsq_rope", _p(x), batch, seq, heads, hd, theta, inverse, _stream(stream))


def lsq_attention_fwd(q, k, v, o, lse, batch: int, seq: int, hq: int, hkv: int, hd: int, stream=None):
    _call("lsq_attention_fwd", _p(q), _p(k), _p(v), _p(o), _p(lse), batch, seq, hq, hkv, hd, _stream(stream))


def lsq_attention_bwd_workspace_size(batch: int, seq: int, hq: int) -> int:
    return int(_fn("lsq_attention_bwd_workspace_size")(batch, seq, hq))


def lsq_attention_bwd(q, k, v, o, lse, d_o, dq, dk, dv, batch: int, seq: int, hq: int, hkv: int, hd: int,
                      workspace, stream=None):
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _call("lsq_attention_bwd", _p(q), _p(k), _p(v), _p(o), _p(lse), _p(d_o), _p(dq), _p(dk), _p(dv), batch, seq,
          hq, hkv, hd, _p(workspace), wsb, _stream(stream))


def lsq_attention_bwd_ex(q, k, v, o, lse, d_o, dq, dk, dv, batch: int, seq: int, hq: int, hkv: int, hd: int,
                         rope_table, workspace, stream=None):
    """lsq_attention_bwd returning the gradients of the unrotated q and k (rope_table from lsq_rope_table)."""
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    fused = hd == 128 and seq <= 512
    _call("lsq_attention_bwd_ex", _p(q), _p(k), _p(v), _p(o), _p(lse), _p(d_o), _p(dq), _p(dk), _p(dv), batch, seq,
          hq, hkv, hd, _p(rope_table), _p(workspace), wsb, _stream(stream),
          launches=3 if (rope_table is None or fused) else 5)


def lsq_swiglu_fwd(g, u, m, n: int, stream=None):
    _call("lsq_swiglu_fwd", _p(g), _p(u), _p(m), n, _stream(stream))


def lsq_swiglu_bwd(dm, g, u, dg, du, n: int, stream=None):
    _call("lsq_swiglu_bwd", _p(dm), _p(g), _p(u), _p(dg), _p(du), n, _stream(stream))


def lsq_embed_gather(ids, table, h, rows: int, d: int, vocab: int, stream=None):
    _call("lsq_embed_gather", _p(ids), _p(table), _p(h), rows, d, vocab, _stream(stream))


def lsq_xent_workspace_size(rows: int) -> int:
    return int(_fn("lsq_xent_workspace_size")(rows))


def lsq_xent_fwd_bwd(logits, ids, batch: int, seq: int, V: int, loss, dlogits, workspace, stream=None):
    wsb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _call("lsq_xent_fwd_bwd", _p(logits), _p(ids), batch, seq, V, _p(loss), _p(dlogits), _p(workspace), wsb,
          _stream(stream))


def lsq_seq_logprob_workspace_size(rows: int) -> int:
    return int(_fn("lsq_seq_logprob_workspace_size")(rows))


def lsq_seq_logprob(logits, ids, batch: int, seq: int, V: int, row_lse, seq_logp, workspace, stream=None):
    _call("lsq_seq_logprob", _p(logits), _p(ids), batch, seq, V, _p(row_lse), _p(seq_logp), _p(workspace),
          _nbytes(workspace), _stream(stream))


def lsq_dpo_loss(policy_logp, ref_logp, npairs: int, beta: float, loss, dseq, stream=None):
    _call("lsq_dpo_loss", _p(policy_logp), _p(ref_logp), npairs, beta, _p(loss), _p(dseq), _stream(stream))


def lsq_seq_logprob_bwd(logits, ids, batch: int, seq: int, V: int, row_lse, dseq, dlogits, stream=None):
    _call("lsq_seq_logprob_bwd", _p(logits), _p(ids), batch, seq, V, _p(row_lse), _p(dseq), _p(dlogits),
          _stream(stream))


def lsq_lora_refresh_bf16(p, p_bf16, n: int, stream=None):
    _call("lsq_lora_refresh_bf16", _p(p), _p(p_bf16), n, _stream(stream))


def lsq_adamw_step(p, g, m, v, p_bf16, n: int, step: int, lr: float, beta1: float, beta2: float, eps: float,
                   weight_decay: float, stream=None):
    _call("lsq_adamw_step", _p(p), _p(g), _p(m), _p(v), _p(p_bf16), n, step, lr, beta1, beta2, eps, weight_decay,
          _stream(stream))


# ---------------------------------------------------------------------------- streaming
_GATHERS = {}  # scheduler handle -> its ctypes callback (kept alive while the scheduler lives)


def lsq_stream_create(n_layers: int, n_slots: int, record_bytes: int, slots: Sequence[int],
                      host_records: Optional[Sequence[int]], compute_stream, copy_stream, shard=None,
                      disk=None) -> int:
    """shard: None, or (rank, world, gather) for the sharded upload, where
    gather(layer, slot, slot_ptr, record_bytes, copy_stream_handle) enqueues the
    completion of the slot on the copy stream (an all-gather) and raises on failure.
    disk: None, or (path, staging buffers, reader threads) for the disk tier
    (host_records None)."""
    sl = (c_void_p * len(slots))(*[_p(s) for s in slots])
    hr = None if host_records is None else (c_void_p * len(host_records))(*[_p(h) for h in host_records])
    path, stg, nthr = None, None, 0
    if disk is not None:
        path = str(disk[0]).encode()
        stg = (c_void_p * len(disk[1]))(*[_p(b) for b in disk[1]])
        nthr = int(disk[2])
    cb = lsq_gather_fn()
    rank = world = 0
    if shard is not None:
        rank, world, fn = shard

        def _gather(user, layer, slot, slot_ptr, nbytes, stream):
            try:
                fn(int(layer), int(slot), int(slot_ptr or 0), int(nbytes), int(stream or 0))
                return 0
            except Exception as e:  # reported through the scheduler's status
                import sys
                print(f"lsq gather callback failed: {e!r}", file=sys.stderr)
                return 1
        cb = lsq_gather_fn(_gather)
    cfg = lsq_stream_cfg(n_layers, n_slots, record_bytes, sl, hr, rank, world, cb, None, path, stg,
                         0 if disk is None else len(disk[1]), nthr)
    out = c_void_p()
    _call("lsq_stream_create", ctypes.byref(cfg), _stream(compute_stream), _stream(copy_stream), ctypes.byref(out))
    if shard is not None:
        _GATHERS[out.value] = cb
    return out.value


_EXPANDING = set()  # schedulers that launch an absmax expansion after every upload


def lsq_stream_set_absmax_expand(st: int, items, slot_bytes: int):
    """items: [(codes_off, params_off, out_off, nb), ...] (byte offsets from a slot's start)."""
    arr = (lsq_absmax_dq_item * max(len(items), 1))(*[lsq_absmax_dq_item(*it) for it in items])
    _call("lsq_stream_set_absmax_expand", st, arr, len(items), slot_bytes)
    if items:
        _EXPANDING.add(st)
    else:
        _EXPANDING.discard(st)


def _with_uploads(st: int, fn):
    """run fn(); count the expansion kernels of the uploads it issued"""
    if st not in _EXPANDING:
        return fn()
    before = lsq_stream_stats(st)[0]
    out = fn()
    LAUNCHES[0] += lsq_stream_stats(st)[0] - before
    return out


def lsq_layer_upload_async(st: int, layer: int, slot: int):
    _with_uploads(st, lambda: _call("lsq_layer_upload_async", st, layer, slot))


def lsq_stream_step(st: int, layer: int, direction: int) -> int:
    out = c_void_p()
    _with_uploads(st, lambda: _call("lsq_stream_step", st, layer, direction, ctypes.byref(out)))
    return out.value


def lsq_stream_simulate(n_layers: int, n_slots: int, steps):
    """steps: [(layer, direction), ...] -> [(kind, layer, slot), ...] (1 release, 2 upload, 3 wait)."""
    n = len(steps)
    layers = (c_int32 * max(n, 1))(*[l for l, _ in steps])
    dirs = (c_int32 * max(n, 1))(*[d for _, d in steps])
    cap = 4 * n * (n_slots + 2) + 16
    acts = (c_int32 * (3 * cap))()
    cnt = c_int32(0)
    _call("lsq_stream_simulate", n_layers, n_slots, n, layers, dirs, acts, cap, ctypes.byref(cnt))
    return [(acts[3 * i], acts[3 * i + 1], acts[3 * i + 2]) for i in range(cnt.value)]


def lsq_stream_stats(st: int):
    a, b, c = c_int64(0), c_int64(0), c_int64(0)
    _call("lsq_stream_stats", st, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    return a.value, b.value, c.value


def lsq_stream_upload_ms(st: int, layer: int) -> float:
    ms = c_float(0)
    _call("lsq_stream_upload_ms", st, layer, ctypes.byref(ms))
    return ms.value


def lsq_stream_time_waits(st: int, capacity: int):
    _call("lsq_stream_time_waits", st, capacity)


def lsq_stream_wait_ms(st: int):
    """-> (forward ms, backward ms, waits kept, waits dropped) since the previous call."""
    f, b, n, d = c_float(0), c_float(0), c_int32(0), c_int32(0)
    _call("lsq_stream_wait_ms", st, ctypes.byref(f), ctypes.byref(b), ctypes.byref(n), ctypes.byref(d))
    return f.value, b.value, n.value, d.value


def lsq_stream_reset(st: int):
    _call("lsq_stream_reset", st)


def lsq_stream_capture_begin(st: int):
    """Bring the copy stream into the capture open on the compute stream (see lsq.h)."""
    _call("lsq_stream_capture_begin", st)


def lsq_stream_capture_end(st: int):
    _call("lsq_stream_capture_end", st)


def lsq_stream_destroy(st: int):
    _EXPANDING.discard(st)
    _call("lsq_stream_destroy", st)
    _GATHERS.pop(st, None)
