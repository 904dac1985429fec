"""The comparison helpers used by the GPU parity tests (CPU only)."""
import numpy as np
import torch

from parity import assert_close, bf16_half_ulp, errors


def test_half_ulp_bounds_bf16_rounding():
    # fp32 values (the kernels round fp32 accumulators to bf16 once)
    x = (np.random.default_rng(0).standard_normal(100000)
         * np.exp2(np.random.default_rng(1).integers(-20, 20, 100000))).astype(np.float32)
    r = torch.tensor(x).to(torch.bfloat16).double().numpy()
    x = x.astype(np.float64)
    assert np.all(np.abs(r - x) <= bf16_half_ulp(x))
    # and it is tight: the largest observed rounding error reaches most of the bound
    assert np.max(np.abs(r - x) / bf16_half_ulp(x)) > 0.99


def test_assert_close_accepts_rounded_exact_values_and_rejects_errors():
    x = np.random.default_rng(2).standard_normal((64, 16)) * 8
    exact_rounded = torch.tensor(x).to(torch.bfloat16).double().numpy()
    assert_close("rounded", exact_rounded, x)
    bad = exact_rounded.copy()
    bad[3, 4] += 0.05
    try:
        assert_close("bad", bad, x)
    except AssertionError:
        pass
    else:
        raise AssertionError("an error of 0.05 beyond rounding was accepted")


def test_errors_reports_relative_frobenius():
    ref = np.ones(100)
    got = ref + 0.01
    ma, rf = errors(got, ref)
    assert abs(ma - 0.01) < 1e-12 and abs(rf - 0.01) < 1e-12
