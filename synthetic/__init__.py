"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module draws random numbers and nothing else: it holds none of the
arithmetic of NF4 quantisation, the LoRA linear or the decoder layer.  Both
sides of every parity test take their inputs from here, so that neither side
has to import the other.

Recipe (the pages never fix the distributions; these are the stated workloads
of the single-linear case and the plainest extension of it to the stacks):

* frozen base weights  W ~ N(0, 0.02^2) in fp32, rounded to bf16 (RNE);
* LoRA A ~ N(0, 1/K_in), LoRA B ~ N(0, 0.01^2), fp32 masters;
* activations / upstream gradients ~ N(0, 1) rounded to bf16;
* token ids uniform on [0, vocab);
* RMSNorm gains = 1 (their initial value in a Llama/Qwen checkpoint).

Every stream is a numpy Philox generator keyed by (seed, stream id), so a
tensor can be regenerated on its own without drawing the ones before it.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import numpy as np
import torch

WEIGHT_SEED = 0   # frozen base weights
LORA_SEED = 1     # LoRA masters
DATA_SEED = 2     # token ids, activations, upstream gradients

BASE_STD = 0.02
LORA_B_STD = 0.01

LINEARS = ("q", "k", "v", "o", "gate", "up", "down")


@dataclasses.dataclass(frozen=True)
class ModelShape:
    """Shape of a Llama/Qwen decoder stack (no biases, pre-norm, SwiGLU)."""
    name: str
    n_layers: int
    d: int          # hidden size
    f: int          # SwiGLU intermediate size
    n_q: int        # query heads
    n_kv: int       # key/value heads
    vocab: int
    theta: float    # RoPE base
    eps: float      # RMSNorm epsilon
    tied: bool      # lm_head shares the embedding matrix
    r: int          # LoRA rank
    alpha: float = 16.0

    @property
    def hd(self) -> int:
        return self.d // self.n_q

    @property
    def kv(self) -> int:
        return self.n_kv * self.hd

    @property
    def s(self) -> float:
        return self.alpha / self.r

    def linear_shapes(self) -> Dict[str, tuple]:
        """(n_out, k_in) of every frozen linear of one decoder layer."""
        d, f, kv = self.d, self.f, self.kv
        return {"q": (d, d), "k": (kv, d), "v": (kv, d), "o": (d, d),
                "gate": (f, d), "up": (f, d), "down": (d, f)}

    def base_params_per_layer(self) -> int:
        return sum(n * k for n, k in self.linear_shapes().values()) + 2 * self.d

    def total_params(self) -> int:
        emb = self.vocab * self.d
        return (self.n_layers * self.base_params_per_layer() + emb
                + (0 if self.tied else emb) + self.d)


# The stacks the workloads name.  eps: 1e-5 for the Llama-style stacks and
# 1e-6 for the Qwen stack; RoPE without frequency scaling.
SMOL = ModelShape("smollm2-135m", 30, 576, 1536, 9, 3, 49152, 1e4, 1e-5, True, 8)
QWEN3B = ModelShape("qwen2.5-3b", 36, 2048, 11008, 16, 2, 151936, 1e6, 1e-6, True, 16)
LLAMA8B = ModelShape("llama-3.1-8b", 32, 4096, 14336, 32, 8, 128256, 5e5, 1e-5, False, 16)
DENSE32B = ModelShape("dense-32b", 64, 5120, 27648, 40, 8, 152064, 1e6, 1e-5, False, 16)
# Small stacks for tests that the fp64 oracle finishes in seconds.
TINY = ModelShape("tiny", 2, 256, 704, 4, 2, 512, 1e4, 1e-5, True, 8)
TINY_UNTIED = ModelShape("tiny-untied", 3, 256, 704, 4, 1, 1000, 5e5, 1e-5, False, 16)

SHAPES = {s.name: s for s in (SMOL, QWEN3B, LLAMA8B, DENSE32B, TINY, TINY_UNTIED)}


def _gen(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=(int(seed) << 32) | int(stream)))


def normal_f32(seed: int, stream: int, shape, std: float = 1.0) -> np.ndarray:
    g = _gen(seed, stream)
    out = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def bf16(x: np.ndarray) -> torch.Tensor:
    """fp32 numpy array -> bf16 CPU tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def uniform_ids(seed: int, stream: int, shape, vocab: int) -> torch.Tensor:
    g = _gen(seed, stream)
    return torch.from_numpy(g.integers(0, vocab, size=shape, dtype=np.int64)).to(torch.int32)


def _stream(layer: int, idx: int) -> int:
    return 1000 + 16 * layer + idx


# ----------------------------------------------------------------------------
# single linear
# ----------------------------------------------------------------------------

def linear_case(M: int, N: int, K: int, r: int, s: float = 2.0, seed: int = 0) -> dict:
    """W [N,K], X [M,K], dY [M,N] bf16; A [r,K], B [N,r] fp32 masters.

    The single-linear workload is M=64, N=K=512, r=8, s=2 at seed 0.
    """
    base = 7919 * seed
    W = bf16(normal_f32(WEIGHT_SEED, base + 1, (N, K), BASE_STD))
    X = bf16(normal_f32(DATA_SEED, base + 2, (M, K)))
    dY = bf16(normal_f32(DATA_SEED, base + 3, (M, N)))
    A = torch.from_numpy(normal_f32(LORA_SEED, base + 4, (r, K), 1.0 / np.sqrt(K)))
    B = torch.from_numpy(normal_f32(LORA_SEED, base + 5, (N, r), LORA_B_STD))
    return {"W": W, "X": X, "dY": dY, "A": A, "B": B, "s": float(s), "r": r}


def bf16_weight(N: int, K: int, stream: int, std: float = BASE_STD, seed: int = WEIGHT_SEED) -> torch.Tensor:
    return bf16(normal_f32(seed, stream, (N, K), std))


# ----------------------------------------------------------------------------
# decoder stack
# ----------------------------------------------------------------------------

def layer_weights(shape: ModelShape, layer: int) -> Dict[str, torch.Tensor]:
    """bf16 frozen weights of one decoder layer, plus the two RMSNorm gains."""
    out = {}
    for i, (name, (n, k)) in enumerate(shape.linear_shapes().items()):
        out[name] = bf16_weight(n, k, _stream(layer, i))
    out["ln1"] = torch.ones(shape.d, dtype=torch.bfloat16)
    out["ln2"] = torch.ones(shape.d, dtype=torch.bfloat16)
    return out


def embeddings(shape: ModelShape) -> Dict[str, torch.Tensor]:
    emb = bf16_weight(shape.vocab, shape.d, 11)
    out = {"embed": emb, "final_norm": torch.ones(shape.d, dtype=torch.bfloat16)}
    out["lm_head"] = emb if shape.tied else bf16_weight(shape.vocab, shape.d, 12)
    return out


def lora_init(shape: ModelShape) -> List[Dict[str, Dict[str, torch.Tensor]]]:
    """fp32 LoRA masters per layer: {name: {"A": [r,K], "B": [N,r]}}."""
    layers = []
    for l in range(shape.n_layers):
        per = {}
        for i, (name, (n, k)) in enumerate(shape.linear_shapes().items()):
            st = _stream(l, i)
            per[name] = {
                "A": torch.from_numpy(normal_f32(LORA_SEED, st, (shape.r, k), 1.0 / np.sqrt(k))),
                "B": torch.from_numpy(normal_f32(LORA_SEED, st + 8, (n, shape.r), LORA_B_STD)),
            }
        layers.append(per)
    return layers


def tokens(shape: ModelShape, batch: int, seq: int, step: int = 0) -> torch.Tensor:
    """int32 token ids [batch, seq]; targets are the ids shifted by one."""
    return uniform_ids(DATA_SEED, 500 + step, (batch, seq), shape.vocab)


# ----------------------------------------------------------------------------
# device-side draws (fast path for full-size workloads; not reproducible by
# the oracle, which uses the numpy streams above)
# ----------------------------------------------------------------------------

def device_normal_bf16(shape, std: float, seed: int, stream: int, device="cuda") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) << 32) | int(stream))
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def device_normal_f32(shape, std: float, seed: int, stream: int, device="cuda") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) << 32) | int(stream))
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std
