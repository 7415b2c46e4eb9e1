"""Acceptance tolerances for floating-point parity against the fp64 oracle.

GEMM / LoRA outputs and gradients: relative Frobenius error <= 5e-3 and max
elementwise error <= 2e-2 x RMS(reference).  The CUDA path multiplies bf16
operands exactly and accumulates in fp32, then rounds the output to bf16
once.  bf16 keeps 8 significant bits, so its unit roundoff is u = 2^-8: one
rounding moves a value by at most 2^-8 ~ 3.9e-3 of itself, and by about
1.6e-3 of itself in RMS (a uniform error over half an ulp, the ulp being
2^-7 to 2^-8 of the value across a binade).  The 5e-3 Frobenius bound leaves
room for that RMS; the 2e-2 x RMS elementwise bound covers the worst-case
rounding of elements up to about five times the RMS.

Every check records what it measured (relative Frobenius error and the worst
element's error as a fraction of its bound) in RECORD; with LSQ_PARITY_LOG
set, tests/conftest.py writes the records of the session to that file as
JSON, so the margins behind each tolerance can be read off a run.
"""
import os

import numpy as np

REL_FRO = 5e-3
MAX_ABS_RMS = 2e-2
U_BF16 = 2.0 ** -8          # unit roundoff of bf16 (8 significant bits, round to nearest)
U_F32 = 2.0 ** -24

RECORD = []


def record(what: str, kind: str, **values):
    RECORD.append({"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "what": what, "kind": kind,
                   **{k: (float(v) if v is not None else None) for k, v in values.items()}})


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
    record(what, "gemm", rel_fro=rf, rel_fro_bound=rel, max_err_over_rms=mx / max(rms, 1e-300),
           max_err_bound=max_rms)
    assert rf <= rel, f"{what}: relative Frobenius error {rf:.3e} > {rel:.1e}"
    assert mx <= max_rms * rms + 1e-30, f"{what}: max error {mx:.3e} > {max_rms:.0e} x RMS {rms:.3e}"


# Elementwise ops (outputs rounded to bf16 once, inputs bf16): error per
# element <= EW_REL |ref| (one bf16 rounding, at most u = 2^-8 ~ 3.9e-3 of the
# value, plus the fp32 arithmetic before it, with a factor 2 of margin) +
# EW_ABS_RMS x RMS(ref), with the same Frobenius bound as the GEMMs.
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
        record(what, "ew-zero", max_abs=mx, max_abs_bound=zero_atol)
        assert mx <= zero_atol, f"{what}: reference is exactly zero, got max |x| = {mx:.3e}"
        return
    rf = rel_fro(got, ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(got - ref)
    bound = ew_rel * np.abs(ref) + ew_abs_rms * rms
    ratio = err / bound
    worst = int(np.argmax(ratio))
    record(what, "ew", rel_fro=rf, rel_fro_bound=rel, max_err_over_bound=float(ratio.flat[worst]))
    assert rf <= rel, f"{what}: relative Frobenius error {rf:.3e} > {rel:.1e}"
    assert np.all(err <= bound), (f"{what}: element {worst} error {err.flat[worst]:.3e} > "
                                  f"{ew_rel:.0e} x |{ref.flat[worst]:.3e}| + {ew_abs_rms:.0e} x RMS {rms:.3e}")


def assert_within_bound(got, ref, bound, rel=REL_FRO, what="", slack=1.0):
    """Element by element |got - ref| <= slack * bound, where `bound` is a
    first-order rounding-error bound of the computation (see attn_bounds.py),
    plus the relative Frobenius bound."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    bound = np.asarray(bound, dtype=np.float64)
    assert got.shape == ref.shape == bound.shape, (what, got.shape, ref.shape, bound.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    nref = float(np.linalg.norm(ref))
    rf = rel_fro(got, ref) if nref > 0 else None
    ratio = err / np.maximum(slack * bound, 1e-300)
    worst = int(np.argmax(ratio))
    record(what, "bound", rel_fro=rf, rel_fro_bound=rel if nref > 0 else None,
           max_err_over_bound=float(ratio.flat[worst]),
           rms_err_over_rms_bound=float(np.sqrt(np.mean(err ** 2)) / max(np.sqrt(np.mean(bound ** 2)), 1e-300)))
    if rf is not None:
        assert rf <= rel, f"{what}: relative Frobenius error {rf:.3e} > {rel:.1e}"
    assert np.all(err <= slack * bound), (f"{what}: element {worst} error {err.flat[worst]:.3e} > bound "
                                          f"{slack * bound.flat[worst]:.3e} (ref {ref.flat[worst]:.3e})")


def check_model_grads(lora, grads, ref_grads, shape, bound, what=""):
    """LoRA gradients of a whole-model step against the oracle's, tensor by
    tensor: relative Frobenius error <= bound, a number or a mapping
    (layer, name, "A"|"B") -> number (bf16_model.tolerance); every tensor must
    also be non-zero.  Records each tensor's error."""
    names = ("q", "k", "v", "o", "gate", "up", "down")
    for l in range(shape.n_layers):
        for n in names:
            for ab in ("A", "B"):
                got = lora.view(grads, l, n, ab).cpu().numpy()
                want = np.asarray(ref_grads[l][n][ab], dtype=np.float64)
                rf = rel_fro(got, want)
                b = bound[(l, n, ab)] if isinstance(bound, dict) else bound
                record(f"{what} layer {l} {n}.{ab}", "model-grad", rel_fro=rf, rel_fro_bound=b,
                       depth=shape.n_layers - l)
                assert np.abs(got).max() > 0, (what, l, n, ab)
                assert rf <= b, (what, l, n, ab, rf, b)
