"""The polynomial exponential the forward uses for part of its softmax
exponentials (sqa_selftest_exp2_poly runs it elementwise), against 2^x in fp64
and against CUDA's own exp2f.  The forward's parity tests cover it inside the
kernel too; this pins its error bound directly.  Also the throughput probe of
the special-function unit's exponential (sqa_selftest_exp2_rate), which stands
behind the derived exp2 roofline of the dh <= 32 kernels."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _run(cuda_lib, x):
    lib = cuda_lib.load_library()
    f = lib.sqa_selftest_exp2_poly
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    xd = x.cuda()
    y = torch.full_like(xd, float("nan"))
    st = f(xd.data_ptr(), y.data_ptr(), xd.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.sqa_last_error()
    torch.cuda.synchronize()
    return y.cpu()


def test_relative_error_bound_over_the_normal_range(cuda_lib):
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.linspace(-125.0, 8.0, 1 << 20), torch.rand(100001, generator=g) * 133.0 - 125.0,
                   torch.tensor([0.0, 0.5, -0.5, 1.0, -1.0, 0.25, 7.999])])
    y = _run(cuda_lib, x).double().numpy()
    exact = np.exp2(x.double().numpy())
    rel = np.abs(y / exact - 1.0)
    assert rel.max() <= 7.6e-5, rel.max()
    # integers are exact up to the polynomial's value at 0
    xi = torch.arange(-120, 9, dtype=torch.float32)
    yi = _run(cuda_lib, xi).double().numpy()
    assert np.abs(yi / np.exp2(xi.double().numpy()) - 1.0).max() <= 7.6e-5


def test_agrees_with_cuda_exp2f(cuda_lib):
    x = torch.linspace(-30.0, 8.0, 200003)
    y = _run(cuda_lib, x)
    ref = torch.exp2(x.cuda()).cpu()
    assert torch.allclose(y, ref, rtol=8e-5, atol=0.0)


def test_underflow_is_clamped_not_wrapped(cuda_lib):
    x = torch.tensor([-126.0, -126.4, -127.0, -150.0, -1e30, float("-inf")])
    y = _run(cuda_lib, x)
    assert torch.isfinite(y).all() and (y >= 0).all() and (y <= 2.0 ** -125).all()


def test_odd_length_and_tail(cuda_lib):
    x = torch.linspace(-3.0, 3.0, 1001)
    y = _run(cuda_lib, x)
    assert not torch.isnan(y).any()
    assert abs(float(y[-1]) / 8.0 - 1.0) <= 7.6e-5


def test_exponential_rate_is_near_the_derived_unit_count(cuda_lib):
    # 16 exponentials per clock per SM; the probe's rate divided by SMs x the
    # SM clock it ran at must come out near 16 (the clock is read from the
    # device's max clock, so a throttled GPU reads low: the bound is loose)
    lib = cuda_lib.load_library()
    f = lib.sqa_selftest_exp2_rate
    f.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    f.restype = ctypes.c_int
    props = torch.cuda.get_device_properties(0)
    sms = props.multi_processor_count
    blocks, iters = sms * 8, 2048
    out = torch.empty(blocks * 256, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        assert f(out.data_ptr(), blocks, iters, stream) == 0, lib.sqa_last_error()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(5):
        f(out.data_ptr(), blocks, iters, stream)
    b.record()
    torch.cuda.synchronize()
    rate = 5 * blocks * 256 * 8 * iters / (a.elapsed_time(b) * 1e-3)
    clock_hz = props.clock_rate * 1e3 if hasattr(props, "clock_rate") else 1.965e9
    per_clk = rate / sms / clock_hz
    assert torch.isfinite(out).all()
    assert 8.0 <= per_clk <= 16.5, per_clk
