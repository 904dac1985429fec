"""Shared comparison helpers for the GPU parity tests.

Tolerances (bf16 inputs, fp32 accumulation, bf16 outputs): relative Frobenius
error <= 5e-3 and max-abs error <= 2e-2 for O, dQ, dK and dV; max-abs <= 1e-3
for lse (natural log, fp32 output).

The outputs are bf16, so an element whose exact value is x cannot be closer
than half a bf16 ulp of x (2^(floor(log2|x|) - 8)); above |x| = 4 that alone
approaches 2e-2, and gradients of heads in large groups reach |x| ~ 10.  The
max-abs bound is therefore applied to the error in excess of that unavoidable
output rounding; the raw max-abs error is reported beside it.
"""
import numpy as np

MAX_ABS = 2e-2
REL_FRO = 5e-3
LSE_ABS = 1e-3


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def bf16_half_ulp(x):
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def assert_close(name, got, ref, max_abs=MAX_ABS, rel_fro=REL_FRO):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    ma, rf = errors(got, ref)
    excess = float(np.max(np.maximum(np.abs(got - ref) - bf16_half_ulp(ref), 0.0))) if got.size else 0.0
    assert excess <= max_abs and rf <= rel_fro, (
        f"{name}: max-abs beyond bf16 output rounding {excess:.3e} (<= {max_abs}), raw max-abs {ma:.3e}, "
        f"rel-Frobenius {rf:.3e} (<= {rel_fro})")
    return ma, rf


def assert_lse_close(name, got, ref, tol=LSE_ABS):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    ma = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert ma <= tol, f"{name}: lse max-abs {ma:.3e} (<= {tol})"
    return ma
