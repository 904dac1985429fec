"""Shared comparison helpers for the GPU parity tests.

Tolerances (bf16 inputs, fp32 accumulation, bf16 outputs): relative Frobenius
error <= 5e-3 and max-abs error <= 2e-2 for O, dQ, dK and dV; max-abs <= 1e-3
for lse (natural log, fp32 output).

The max-abs bound is applied as stated to every element whose exact value is
below 4 in magnitude.  Where |x| >= 4 the output format alone takes most of
it: the nearest bf16 number can be half a bf16 ulp away, 2^(floor(log2|x|) - 8),
which is 0.0156 in [4, 8) and 0.031 in [8, 16) (gradients of heads in large
groups reach |x| ~ 10-17).  Only there the bound is applied to the error in
excess of that half ulp.

Every comparison is appended as one JSON line to the file named by the
environment variable SQA_PARITY_LOG, when it is set, so that the raw errors of
passing tests are on record too.
"""
import json
import os

import numpy as np

MAX_ABS = 2e-2
REL_FRO = 5e-3
LSE_ABS = 1e-3
# |exact| from which the half-ulp allowance for bf16 output rounding applies
LARGE = 4.0


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


def split_errors(got, ref):
    """(largest error where |ref| < LARGE, largest error beyond half a bf16 ulp where |ref| >= LARGE)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    small = np.abs(ref) < LARGE
    raw_small = float(np.max(err[small])) if np.any(small) else 0.0
    big = ~small
    excess_big = float(np.max(err[big] - bf16_half_ulp(ref[big]))) if np.any(big) else 0.0
    return raw_small, excess_big


def record(entry):
    path = os.environ.get("SQA_PARITY_LOG")
    if not path:
        return
    entry = dict(entry, test=os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0])
    with open(path, "a") as f:
        f.write(json.dumps(entry) + "\n")


def assert_close(name, got, ref, max_abs=MAX_ABS, rel_fro=REL_FRO):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    ma, rf = errors(got, ref)
    raw_small, excess_big = split_errors(got, ref)
    max_ref = float(np.max(np.abs(ref))) if ref.size else 0.0
    record({"name": name, "max_abs": ma, "max_abs_below_4": raw_small, "excess_at_4_and_above": excess_big,
            "rel_fro": rf, "max_abs_ref": max_ref, "n": int(ref.size)})
    assert raw_small <= max_abs and excess_big <= max_abs and rf <= rel_fro, (
        f"{name}: max-abs {raw_small:.3e} where |ref| < {LARGE} (<= {max_abs}), "
        f"beyond half a bf16 ulp {excess_big:.3e} where |ref| >= {LARGE} (<= {max_abs}), raw max-abs {ma:.3e}, "
        f"rel-Frobenius {rf:.3e} (<= {rel_fro}), max |ref| {max_ref:.3g}")
    return ma, rf


def assert_lse_close(name, got, ref, tol=LSE_ABS):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    ma = float(np.max(np.abs(got - ref))) if got.size else 0.0
    record({"name": name, "lse_max_abs": ma, "n": int(got.size)})
    assert ma <= tol, f"{name}: lse max-abs {ma:.3e} (<= {tol})"
    return ma


# The full layer and the decoder block keep their intermediates in bf16 (see
# tests/test_layer_gpu.py for the derivation): relative Frobenius <= 1e-2 and,
# element by element, |error| <= 2e-2 + 0.1 * RMS(exact).
SCALED_REL_FRO = 1e-2


def assert_scaled_close(name, got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bound = 2e-2 + 0.1 * rms
    rf = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    record({"name": name, "max_abs": float(err.max()), "rms_ref": rms, "rel_fro": rf, "n": int(ref.size)})
    assert err.max() <= bound and rf <= SCALED_REL_FRO, (
        f"{name}: max-abs {err.max():.3e} (<= {bound:.3e}), rel-Frobenius {rf:.3e} (<= {SCALED_REL_FRO})")
