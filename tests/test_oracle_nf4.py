"""Pins for the oracle's NF4 quantiser (CPU only).

Each pin checks the oracle against something other than itself: the closed-form
construction with an independent inverse-normal routine, a pure-Python brute
force, the exact round trip, and torch's own fp32 -> bf16 rounding.
"""
import json
import os

import numpy as np
import pytest
import torch
from scipy.special import ndtr, ndtri

from oracle import nf4
import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_codebook_invariants():
    cb = nf4.codebook()
    assert cb.dtype == np.float32 and cb.shape == (16,)
    assert np.all(np.diff(cb.astype(np.float64)) > 0)
    assert cb[0] == -1.0 and cb[15] == 1.0
    assert cb[7] == 0.0 and not np.signbit(cb[7])
    assert (cb > 0).sum() == 8 and (cb < 0).sum() == 7


def test_codebook_matches_library_inverse_normal():
    # the same construction through scipy's ndtri: an independent Phi^-1
    d = nf4.DELTA
    pos = ndtri(np.linspace(d, 0.5, 9)[:-1])
    neg = -ndtri(np.linspace(d, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, neg, [0.0]]))
    v = (v / v.max()).astype(np.float32)
    assert np.array_equal(v.view(np.uint32), nf4.codebook().view(np.uint32))


def test_codebook_levels_are_normal_quantiles():
    # c_i * Phi^-1(delta) must sit at the evenly spaced probabilities
    cb = nf4.codebook_f64()
    top = ndtri(nf4.DELTA)
    p_pos = ndtr(cb[8:] * top)
    np.testing.assert_allclose(np.sort(p_pos)[::-1], np.linspace(nf4.DELTA, 0.5, 9)[:-1], rtol=0, atol=1e-12)
    p_neg = ndtr(-cb[:7] * top)
    np.testing.assert_allclose(np.sort(p_neg)[::-1], np.linspace(nf4.DELTA, 0.5, 8)[:-1], rtol=0, atol=1e-12)


def _brute_code(x, cb):
    best, bi = None, None
    for i, c in enumerate(cb.astype(float)):
        d = abs(float(x) - c)
        if best is None or d < best:       # strict: ties keep the lower index
            best, bi = d, i
    return bi


def test_quantize_brute_force_small():
    w = S.bf16_weight(3, 128, stream=77).float().numpy()
    codes, am = nf4.quantize_codes(w)
    cb = nf4.codebook()
    for n in range(3):
        for b in range(2):
            blk = w[n, 64 * b: 64 * (b + 1)]
            a = max(abs(float(t)) for t in blk)
            assert np.float32(a) == am[n, b]
            for j, t in enumerate(blk):
                x = np.float32(np.float32(t) / np.float32(a))
                assert codes[n, 64 * b + j] == _brute_code(x, cb)


def test_quantize_zero_block_and_signed_zero():
    w = np.zeros((2, 128), dtype=np.float32)
    w[1, 64:] = np.linspace(-1, 1, 64, dtype=np.float32)
    w[1, 70] = -0.0
    codes, am = nf4.quantize_codes(w)
    assert np.all(codes[0] == nf4.ZERO_CODE) and np.all(am[0] == 0)
    assert np.all(codes[1, :64] == nf4.ZERO_CODE)
    assert codes[1, 70] == nf4.ZERO_CODE
    assert codes[1, 64] == 0 and codes[1, 127] == 15


def test_decision_boundaries_are_midpoints_ties_low():
    cb = nf4.codebook()
    for i in range(15):
        mid = (float(cb[i]) + float(cb[i + 1])) / 2.0          # exact in fp64
        m32 = np.float32(mid)
        below = m32 if float(m32) < mid else np.nextafter(m32, np.float32(-2))
        above = m32 if float(m32) > mid else np.nextafter(m32, np.float32(2))
        got = nf4.nearest_code(np.array([below, above], np.float32))
        assert got.tolist() == [i, i + 1]
        if float(m32) == mid:                                # an exact tie
            assert nf4.nearest_code(np.array([m32]))[0] == i


def test_round_trip_exact():
    rng = np.random.default_rng(5)
    N, K = 8, 256
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    blocks = codes.reshape(N, K // 64, 64)
    blocks[:, :, 0] = rng.choice([0, 15], size=(N, K // 64))   # each block holds +-1
    a = nf4.bf16_round(rng.uniform(1e-3, 2.0, size=(N, K // 64)).astype(np.float32))
    packed = nf4.pack(codes)
    wq = nf4.dequantize(packed, a, N, K)
    w = nf4.bf16_bits_to_f32(wq)
    p2, a2 = nf4.quantize(w)
    assert np.array_equal(a2, a)
    assert np.array_equal(p2, packed)
    assert np.array_equal(nf4.dequantize(p2, a2, N, K), wq)


def test_pack_high_nibble_first():
    c = np.array([1, 2, 15, 0, 7, 7], dtype=np.uint8)
    assert nf4.pack(c).tolist() == [0x12, 0xF0, 0x77]
    assert nf4.unpack(nf4.pack(c)).tolist() == c.tolist()


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(100000).astype(np.float32) * np.float32(3.0)
    # add exact ties: values halfway between two bf16 numbers
    ties = ((rng.integers(0, 1 << 15, 1000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties[np.isfinite(ties)]])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(nf4.f32_to_bf16_bits(x), ref)


def test_dequant_is_one_fp32_multiply_then_bf16():
    cb = nf4.codebook()
    codes = np.arange(16, dtype=np.uint8).repeat(4)    # 64 codes = one block
    a = np.array([[0.0371]], dtype=np.float32)
    got = nf4.bf16_bits_to_f32(nf4.dequantize(nf4.pack(codes), a, 1, 64))[0]
    for j, c in enumerate(codes):
        want = torch.tensor(float(np.float32(cb[c]) * np.float32(0.0371)), dtype=torch.float32).to(torch.bfloat16).float().item()
        assert got[j] == np.float32(want)


def test_param_count_golden():
    with open(os.path.join(GOLDEN, "smollm2_135m_param_count.json")) as f:
        g = json.load(f)
    assert S.SMOL.total_params() == g["value"]
