"""Pins for the oracle's double-quantised absmax (CPU only).

* the E4M3 value table against torch's float8_e4m3fn type (a library
  decoding of the same format) and against the format's closed-form facts;
* E4M3 rounding against torch's conversion on random values and on every
  midpoint between neighbouring codes (ties to even);
* blocks built from representable values round-trip exactly (codes,
  centre, scale and the expanded absmax);
* on absmax arrays shaped like the workloads' the expansion error stays
  inside the E4M3 half-ulp bound, block extremes land on +-448, constant and
  all-zero blocks are exact, ragged last blocks are handled;
* the 8B layer record then comes to the pages' 113 MB buffer size.
"""
import math

import numpy as np
import pytest
import torch

import synthetic as S
from oracle import nf4

F32 = np.float32


def _canon(codes):
    """negative zero (0x80) is stored as +0"""
    c = np.array(codes, dtype=np.uint8)
    c[c == 0x80] = 0
    return c


def test_e4m3_table_matches_torch():
    mine = nf4.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])


def test_e4m3_table_closed_form():
    t = nf4.e4m3_table()
    pos = t[:0x7F]
    assert pos[0] == 0.0 and pos[1] == 2.0 ** -9 and pos[8] == 2.0 ** -6 and pos[-1] == 448.0
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(t[0x80:0xFF], -pos)
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    # 3 mantissa bits: neighbours among the normal values differ by at most 1/8 of the smaller
    assert np.all(np.diff(pos[8:]) <= pos[8:-1] / 8 + 1e-300)


def test_e4m3_round_matches_torch_random():
    g = np.random.default_rng(0)
    x = np.concatenate([g.uniform(-448, 448, 20000), g.normal(0, 1, 20000), g.normal(0, 1e-2, 5000)]).astype(F32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nf4.e4m3_round(x), _canon(ref))


def test_e4m3_round_ties_to_even():
    pos = nf4.e4m3_table()[:0x7F]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(F32)          # every midpoint is an exact fp32
    assert np.array_equal(mids.astype(np.float64), (pos[:-1] + pos[1:]) / 2)
    codes = nf4.e4m3_round(mids)
    lower = np.arange(0x7E)
    want = np.where(lower % 2 == 0, lower, lower + 1)
    assert np.array_equal(codes, want.astype(np.uint8))
    ref = torch.from_numpy(np.concatenate([mids, -mids])).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nf4.e4m3_round(np.concatenate([mids, -mids])), _canon(ref))
    # saturation and signed zero
    sat = nf4.e4m3_round(np.array([449.0, 1e30, -1e30, -1e-7, 0.0, -0.0], dtype=F32))
    assert list(sat) == [0x7E, 0x7E, 0xFE, 0, 0, 0]


def test_double_quant_exact_on_representable_blocks():
    g = np.random.default_rng(1)
    tab = nf4.e4m3_table()
    for trial in range(20):
        n = int(g.integers(1, 4)) * 256 + int(g.integers(0, 256))
        # coarse centre and power-of-two scale: every c + v * s is an exact fp32
        centre = F32(int(g.integers(20, 200)) / 1024)
        scale = F32(2.0 ** int(g.integers(-17, -13)))
        codes = g.integers(0, 0x7F, n).astype(np.uint8) | (g.integers(0, 2, n).astype(np.uint8) << 7)
        codes[codes == 0x80] = 0
        codes[codes == 0xFF] = 0xFE
        for b in range(0, n, 256):                          # every block holds both extremes
            codes[b] = 0x7E
            if b + 1 < n:
                codes[b + 1] = 0xFE
        a = (centre + tab[codes] * float(scale)).astype(F32)
        assert np.array_equal(a.astype(np.float64), float(centre) + tab[codes] * float(scale))  # exact
        q, p = nf4.double_quantize_absmax(a)
        full = [b for b in range(0, n, 256) if b + 1 < n]
        assert np.array_equal(p[[b // 256 for b in full]], np.array([[centre, scale]] * len(full), dtype=F32))
        last = n - 1
        if last % 256 == 0:                                 # a one-value last block is constant
            assert q[last] == 0 and p[-1, 1] == 0
            q, codes = q[:last], codes[:last]
        assert np.array_equal(q, codes)
        assert np.array_equal(nf4.double_quantized(a), a)


def _workload_absmax(n_blocks, seed):
    """absmax of N(0, 0.02) weights in blocks of 64, as the quantiser sees them"""
    w = S.normal_f32(S.WEIGHT_SEED, seed, (n_blocks, 64), S.BASE_STD)
    return nf4.bf16_round(np.abs(w)).max(axis=1).astype(F32)


@pytest.mark.parametrize("n", [256, 1000, 4096 + 17])
def test_double_quant_error_bound_and_extremes(n):
    a = _workload_absmax(n, 5 + n)
    q, p = nf4.double_quantize_absmax(a)
    e = nf4.expand_absmax(q, p)
    for b in range(p.shape[0]):
        blk = a[b * 256:(b + 1) * 256]
        centre, scale = p[b]
        half = float(np.float32(blk.max() - blk.min()) * 0.5)
        # E4M3 keeps 3 mantissa bits: half an ulp is at most 2^-4 of the value
        # (normal range) and 2^-10 * scale absolute (subnormal range); the two
        # fp32 roundings of the expansion add a few ulp of the result
        bound = half * 2.0 ** -4 + scale * 2.0 ** -10 + 4 * np.spacing(blk.max())
        assert np.max(np.abs(e[b * 256:(b + 1) * 256].astype(np.float64) - blk)) <= bound
        if blk.max() > blk.min():
            assert q[b * 256 + int(np.argmax(blk))] == 0x7E
            assert q[b * 256 + int(np.argmin(blk))] == 0xFE
    # absmax of N(0, sigma) blocks of 64 spread about +-25% around their centre, so the
    # expanded scale is within about 2% of the exact one (NF4 levels are 7-30% apart)
    assert np.max(np.abs(e - a) / a) < 3e-2


def test_double_quant_constant_and_zero_blocks():
    a = np.concatenate([np.full(256, 0.0371, F32), np.zeros(256, F32), np.full(7, 0.5, F32)])
    q, p = nf4.double_quantize_absmax(a)
    assert np.all(q == 0) and np.all(p[:, 1] == 0)
    assert np.array_equal(nf4.expand_absmax(q, p), a)


def test_double_quant_footprint_matches_pages_buffer_size():
    """The pages size the 8B layer buffers at 113 MB (README layer-streaming
    figure); with fp32 absmax the same record is 122.7 MB."""
    sh = S.SHAPES["llama-3.1-8b"]
    codes = sum(n * k // 2 for n, k in sh.linear_shapes().values())
    blocks = [n * k // 64 for n, k in sh.linear_shapes().values()]
    dq = codes + sum(b + 8 * math.ceil(b / 256) for b in blocks) + 2 * 2 * sh.d
    fp32 = codes + sum(4 * b for b in blocks) + 2 * 2 * sh.d
    assert abs(dq / 1e6 - 113) < 1.0, dq
    assert abs(fp32 / 1e6 - 122.7) < 0.1, fp32
