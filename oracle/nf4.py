"""NF4 blockwise quantisation written out from its definition (oracle).

TEST INFRASTRUCTURE ONLY: see ``oracle/__init__.py``.

What the pages fix: the frozen base is quantised once, offline, one tensor at a
time, to "NF4", and the streamed bytes are the quantised bytes (soup-cli
0.72.0 -> 0.72.2 diff, CHANGELOG [0.72.2] "Added - NF4 layer streaming" and
docs/performance-and-quantization.md "NF4 streaming (quantization: 4bit)").

Readings taken where they are silent:
* codebook: the published NormalFloat-4 construction (Dettmers et al., QLoRA
  2023, sec. 3): 8 positive normal quantiles at probabilities evenly spaced
  from delta to 1/2 (9 points, the 1/2 point dropped), 7 negative ones from 8
  points, an exact 0, sorted and divided by the largest; delta =
  1 - (1/30 + 1/32)/2.  Values in fp64, then rounded to fp32.
* block = 64 consecutive elements of the row-major tensor (every K_in of the
  workloads is a multiple of 64, so a block never straddles two rows);
  absmax = max |w| of the block in fp32, stored row-major [N, K/64].
* x = w / absmax in fp32 (IEEE division, round to nearest even).
* code = argmin_i |x - c_i|, exact (fp64 on fp32 operands); ties go to the
  lower index; an all-zero block stores absmax 0 and every code 7 (the zero).
* packing: byte j = (code[2j] << 4) | code[2j+1] (first element, high nibble).
* dequant: w' = bf16_rn( fp32(c[code]) * absmax ) - one fp32 multiply, then
  round to nearest even to bf16.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64
DELTA = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
ZERO_CODE = 7


def _normal_cdf(x: float) -> float:
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def inverse_normal_cdf(p: float) -> float:
    """Phi^-1(p) by bisection on the erfc-based CDF until the bracket is one ulp."""
    lo, hi = -40.0, 40.0
    while True:
        mid = 0.5 * (lo + hi)
        if mid <= lo or mid >= hi:
            break
        if _normal_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    # the two ends of the final bracket: keep the one whose CDF is nearer p
    return lo if abs(_normal_cdf(lo) - p) <= abs(_normal_cdf(hi) - p) else hi


def codebook_f64(delta: float = DELTA) -> np.ndarray:
    pos = [inverse_normal_cdf(p) for p in np.linspace(delta, 0.5, 9)[:-1]]
    neg = [-inverse_normal_cdf(p) for p in np.linspace(delta, 0.5, 8)[:-1]]
    vals = np.array(sorted(pos + neg + [0.0]), dtype=np.float64)
    return vals / vals.max()


def codebook() -> np.ndarray:
    """The 16 NF4 levels as fp32, ascending; index 7 is exactly 0."""
    return codebook_f64().astype(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    out = b.astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16, returned as fp32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


def absmax_blocks(w: np.ndarray) -> np.ndarray:
    """absmax per 64-element block of a row-major [N, K] tensor -> fp32 [N, K/64]."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % BLOCK == 0, "K_in must be a multiple of the block size"
    return np.abs(w.reshape(N, K // BLOCK, BLOCK)).max(axis=2).astype(np.float32)


def nearest_code(x: np.ndarray, cb: np.ndarray | None = None) -> np.ndarray:
    """argmin_i |x - c_i| over the 16 levels, ties to the lower index (brute force)."""
    cb = codebook() if cb is None else cb
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    out = np.empty(x.shape, dtype=np.uint8)
    c64 = cb.astype(np.float64)
    step = 1 << 20
    for i in range(0, x.size, step):
        xs = x[i:i + step].astype(np.float64)
        dist = np.abs(xs[:, None] - c64[None, :])
        out[i:i + step] = np.argmin(dist, axis=1)   # first minimum = lower index
    return out


def quantize_codes(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16-valued [N, K] -> (codes uint8 [N, K] one per element, absmax fp32 [N, K/64])."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    am = absmax_blocks(w)
    blocks = w.reshape(N, K // BLOCK, BLOCK)
    denom = np.where(am == 0, np.float32(1), am)[:, :, None].astype(np.float32)
    x = (blocks / denom).astype(np.float32)          # IEEE fp32 division
    codes = nearest_code(x).reshape(N, K // BLOCK, BLOCK)
    codes[am == 0] = ZERO_CODE
    return codes.reshape(N, K), am


def pack(codes: np.ndarray) -> np.ndarray:
    """two codes per byte, first element in the high nibble -> uint8 [numel/2]."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, 2)
    return ((c[:, 0] << 4) | c[:, 1]).astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 0x0F
    return out


def quantize(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """bf16-valued [N, K] -> (packed uint8 [N*K/2], absmax fp32 [N, K/64])."""
    codes, am = quantize_codes(w)
    return pack(codes), am


def dequantize(packed: np.ndarray, absmax: np.ndarray, N: int, K: int) -> np.ndarray:
    """-> bf16 bit patterns uint16 [N, K]: bf16_rn(fp32(c[code]) * absmax)."""
    cb = codebook()
    codes = unpack(packed).reshape(N, K // BLOCK, BLOCK)
    am = np.asarray(absmax, dtype=np.float32).reshape(N, K // BLOCK, 1)
    prod = (cb[codes] * am).astype(np.float32)       # one fp32 multiply, RN
    return f32_to_bf16_bits(prod).reshape(N, K)


def dequantize_f64(packed: np.ndarray, absmax: np.ndarray, N: int, K: int) -> np.ndarray:
    return bf16_bits_to_f32(dequantize(packed, absmax, N, K)).astype(np.float64)
