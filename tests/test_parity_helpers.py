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


def test_max_abs_bound_is_raw_below_four_and_over_rounding_above():
    ref = np.array([3.0, 5.0, 10.0, -0.5])
    # below |x| = 4 the stated bound applies to the raw error
    for err, ok in ((0.019, True), (0.021, False)):
        got = ref.copy()
        got[0] += err
        try:
            assert_close("small", got, ref, rel_fro=1.0)
            accepted = True
        except AssertionError:
            accepted = False
        assert accepted == ok, err
    # at |x| = 5 half a bf16 ulp is 2^-6 = 0.015625: 0.03 raw is 0.0144 beyond it
    for err, ok in ((0.03, True), (0.04, False)):
        got = ref.copy()
        got[1] += err
        try:
            assert_close("large", got, ref, rel_fro=1.0)
            accepted = True
        except AssertionError:
            accepted = False
        assert accepted == ok, err


def test_comparisons_are_logged(tmp_path, monkeypatch):
    import json

    from parity import assert_lse_close

    log = tmp_path / "parity.jsonl"
    monkeypatch.setenv("SQA_PARITY_LOG", str(log))
    assert_close("out", np.array([1.0, 2.01]), np.array([1.0, 2.0]))
    assert_lse_close("lse", np.array([0.5]), np.array([0.5002]))
    rows = [json.loads(l) for l in log.read_text().splitlines()]
    assert rows[0]["name"] == "out" and abs(rows[0]["max_abs"] - 0.01) < 1e-12
    assert rows[0]["max_abs_below_4"] == rows[0]["max_abs"] and rows[0]["excess_at_4_and_above"] == 0.0
    assert rows[1]["name"] == "lse" and abs(rows[1]["lse_max_abs"] - 2e-4) < 1e-12
