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


# ------------------------------------------------------------------------
# Double quantisation of the absmax array (8-bit second level).
#
# The pages give only its footprint: the 8B base store at 3.60 GB and layer
# buffers of 113 MB ("Soup" README, layer-streaming figure caption and the
# 8B row of its benchmark table), which is what 4-bit codes plus roughly one
# byte per 64-element block come to, not the 4 bytes of an fp32 absmax.  The
# construction is the QLoRA paper's "double quantization" (Dettmers et al.
# 2023, sec. 3): the first-level constants are themselves quantised to 8-bit
# floats in blocks of 256, after centring.  Readings taken where that text
# leaves the details open:
# * 8-bit float = E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa
#   bits, exponent field 0 subnormal, no infinities, S.1111.111 the only NaN;
#   largest finite 448);
# * block = 256 consecutive absmax values of one tensor (row-major [N, K/64]
#   flattened; the last block of a tensor may be shorter);
# * centring and scale per block: centre = fp32(fp32(hi + lo) * 0.5), half =
#   fp32(fp32(hi - lo) * 0.5), scale = fp32(half / 448) (lo, hi: the block's
#   smallest and largest absmax), so the block's extremes land on -448 and
#   +448;
# * code = the E4M3 value nearest to fp32(fp32(a - centre) / scale), ties to
#   the even code, magnitudes beyond 448 saturating to 448, a zero result
#   stored as +0 (code 0); a block with scale 0 stores every code 0;
# * expansion: a' = fp32(fp32(e4m3(code) * scale) + centre), two roundings.
# ------------------------------------------------------------------------
DQ_BLOCK = 256
E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """Value of one E4M3 bit pattern, from the field definitions."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    """float64 [256]: the value of every code (NaN at 0x7F and 0xFF)."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code to each fp32 value (brute force over the 127
    non-negative finite codes, distances exact in fp64); ties go to the even
    code; magnitudes above 448 end on 448 (the nearest finite value); a result
    of zero is +0."""
    x = np.asarray(x, dtype=np.float32).reshape(-1)
    mags = e4m3_table()[:0x7F]                      # codes 0..126, increasing
    # saturate first: every magnitude at or above 448 takes the largest finite code
    # (this also keeps the distances below exact in fp64)
    a = np.minimum(np.abs(x.astype(np.float64)), E4M3_MAX)
    dist = np.abs(a[:, None] - mags[None, :])
    best = dist.min(axis=1, keepdims=True)
    tied = dist == best
    # among the (at most two, adjacent) nearest codes prefer the even one
    even = tied & ((np.arange(0x7F) % 2) == 0)[None, :]
    code = np.where(even.any(axis=1), even.argmax(axis=1), tied.argmax(axis=1)).astype(np.uint8)
    neg = (x < 0) & (code != 0)
    code[neg] |= 0x80
    return code


def double_quantize_absmax(absmax: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """fp32 absmax (any shape, row-major) -> (codes uint8 [n], params fp32
    [ceil(n / 256), 2] holding (centre, scale) per block of 256)."""
    a = np.asarray(absmax, dtype=np.float32).reshape(-1)
    n = a.size
    nblk = (n + DQ_BLOCK - 1) // DQ_BLOCK
    codes = np.zeros(n, dtype=np.uint8)
    params = np.zeros((nblk, 2), dtype=np.float32)
    half_f, max_f = np.float32(0.5), np.float32(E4M3_MAX)
    for b in range(nblk):
        blk = a[b * DQ_BLOCK:(b + 1) * DQ_BLOCK]
        lo, hi = blk.min(), blk.max()
        centre = np.float32(np.float32(hi + lo) * half_f)
        half = np.float32(np.float32(hi - lo) * half_f)
        scale = np.float32(half / max_f)
        params[b] = (centre, scale)
        if scale != 0:
            x = ((blk - centre).astype(np.float32) / scale).astype(np.float32)
            codes[b * DQ_BLOCK:b * DQ_BLOCK + blk.size] = e4m3_round(x)
    return codes, params


def expand_absmax(codes: np.ndarray, params: np.ndarray) -> np.ndarray:
    """(codes, (centre, scale) per 256) -> fp32 absmax [n]: fp32(fp32(e4m3 * scale) + centre)."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1)
    p = np.asarray(params, dtype=np.float32).reshape(-1, 2)
    blk = np.arange(c.size) // DQ_BLOCK
    v = e4m3_table()[c].astype(np.float32)           # exact: every E4M3 value is an fp32
    prod = (v * p[blk, 1]).astype(np.float32)
    return (prod + p[blk, 0]).astype(np.float32)


def double_quantized(absmax: np.ndarray) -> np.ndarray:
    """The absmax a double-quantised store hands to the dequantiser: expand(quantise(absmax)), same shape."""
    am = np.asarray(absmax, dtype=np.float32)
    return expand_absmax(*double_quantize_absmax(am)).reshape(am.shape)
