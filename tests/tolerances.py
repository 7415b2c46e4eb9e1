"""Acceptance tolerances for floating-point parity against the fp64 oracle.

GEMM / LoRA outputs and gradients: relative Frobenius error <= 5e-3 and max
elementwise error <= 2e-2 x RMS(reference).  The CUDA path multiplies bf16
operands exactly and accumulates in fp32, then rounds the output to bf16
once: the bf16 rounding alone is a relative error of at most 2^-9 ~ 2e-3 per
element, which is what the 5e-3 Frobenius bound leaves room for.
"""
import numpy as np

REL_FRO = 5e-3
MAX_ABS_RMS = 2e-2


def rel_fro(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_close(got, ref, rel=REL_FRO, max_rms=MAX_ABS_RMS, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rf = rel_fro(got, ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    mx = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert rf <= rel, f"{what}: relative Frobenius error {rf:.3e} > {rel:.1e}"
    assert mx <= max_rms * rms + 1e-30, f"{what}: max error {mx:.3e} > {max_rms:.0e} x RMS {rms:.3e}"


# Elementwise ops and attention (outputs rounded to bf16 once, inputs bf16):
# error per element <= EW_REL |ref| (a bf16 ulp is 2^-8 relative, rounding
# half of it, plus fp32 arithmetic) + EW_ABS_RMS x RMS(ref), with the same
# Frobenius bound as the GEMMs.
EW_REL = 8e-3
EW_ABS_RMS = 2e-2


def assert_close_ew(got, ref, rel=REL_FRO, ew_rel=EW_REL, ew_abs_rms=EW_ABS_RMS, what="", zero_atol=1e-6):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    nref = float(np.linalg.norm(ref))
    if nref == 0.0:
        mx = float(np.max(np.abs(got))) if got.size else 0.0
        assert mx <= zero_atol, f"{what}: reference is exactly zero, got max |x| = {mx:.3e}"
        return
    rf = rel_fro(got, ref)
    assert rf <= rel, f"{what}: relative Frobenius error {rf:.3e} > {rel:.1e}"
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(got - ref)
    bound = ew_rel * np.abs(ref) + ew_abs_rms * rms
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), (f"{what}: element {worst} error {err.flat[worst]:.3e} > "
                                  f"{ew_rel:.0e} x |{ref.flat[worst]:.3e}| + {ew_abs_rms:.0e} x RMS {rms:.3e}")


# Attention gradients: a row of dQ (one query, one head) sums dS_ij K_j over its
# keys with dS in bf16, so its error scales with the row's own magnitude (rows
# of early positions, with few keys and concentrated probabilities, are much
# larger than the average).  Per row (last axis): ||err|| <= ROW_REL ||ref row||
# + ROW_FLOOR x RMS(ref) x sqrt(row length), plus the Frobenius bound.
ROW_REL = 2e-2
ROW_FLOOR = 2e-2


def assert_close_rows(got, ref, rel=1e-2, row_rel=ROW_REL, row_floor=ROW_FLOOR, what="", zero_atol=1e-4):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    nref = float(np.linalg.norm(ref))
    if nref == 0.0:
        mx = float(np.max(np.abs(got))) if got.size else 0.0
        assert mx <= zero_atol, f"{what}: reference is exactly zero, got max |x| = {mx:.3e}"
        return
    rf = rel_fro(got, ref)
    assert rf <= rel, f"{what}: relative Frobenius error {rf:.3e} > {rel:.1e}"
    n = ref.shape[-1]
    g2, r2 = got.reshape(-1, n), ref.reshape(-1, n)
    err = np.linalg.norm(g2 - r2, axis=1)
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = row_rel * np.linalg.norm(r2, axis=1) + row_floor * rms * np.sqrt(n)
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), (f"{what}: row {worst} error {err[worst]:.3e} > {row_rel:.0e} x "
                                  f"{np.linalg.norm(r2[worst]):.3e} + {row_floor:.0e} x RMS {rms:.3e} x sqrt({n})")
