"""Failure detection and stray writes, tested without faulting or hanging a GPU.

* Bounded waits: sqa_selftest_wait_timeout runs the kernels' bounded mbarrier
  wait on a barrier that nothing completes, with a limit of a millisecond.  The
  device status word must then carry the site's bit, the timeout record must
  name the give-up (block 0, the site, thread 0, parity 0), the kernel must
  have returned, and the context must still run the attention kernels.
* Canaries: every output buffer of the forward, backward, decoding step and
  layer is placed between guard regions filled with a byte pattern, at ragged
  sizes; after the call the guards must be untouched and every output element
  written (the interior starts as NaN).
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_query_attention_sqa_b200.inputs import make_decode_inputs, make_inputs, make_layer_inputs

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side; keeps the interior 256-byte aligned
PATTERN = 0xA5


def _selftest(lib, limit_us, site):
    f = lib.sqa_selftest_wait_timeout
    f.argtypes = [ctypes.c_uint, ctypes.c_uint, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f(limit_us, site, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("site", [0, 2, 3])
def test_bounded_wait_gives_up_and_reports(cuda_lib, site):
    lib = cuda_lib.load_library()
    cuda_lib.device_status(clear=True)
    cuda_lib.timeout_info(clear=True)
    assert _selftest(lib, 1000, site) == 0
    torch.cuda.synchronize()  # the kernel returned
    assert cuda_lib.device_status(clear=True) == 1 << site
    info = cuda_lib.timeout_info(clear=True)
    assert info is not None and info["block"] == 0 and info["role"] == site
    assert info["thread"] == 0 and info["parity"] == 0
    assert cuda_lib.device_status() == 0 and cuda_lib.timeout_info() is None
    # the context still runs the attention kernels correctly
    q, k, v, _ = make_inputs(1, 200, 8, 4, 16, seed=1)
    out, lse = cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_bounded_wait_selftest_rejects_bad_arguments(cuda_lib):
    lib = cuda_lib.load_library()
    assert _selftest(lib, 0, 0) == cuda_lib.SQA_ERR_INVALID_ARG
    assert _selftest(lib, 200000, 0) == cuda_lib.SQA_ERR_INVALID_ARG
    assert _selftest(lib, 1000, 5) == cuda_lib.SQA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0


class Guarded:
    """A CUDA tensor of `shape`/`dtype` inside a byte buffer with guard regions."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(*shape)
        if dtype.is_floating_point:
            self.t.fill_(float("nan"))
        else:
            self.t.fill_(0)

    def check(self, name):
        torch.cuda.synchronize()
        assert bool((self.raw[:GUARD] == PATTERN).all()), f"{name}: write before the buffer"
        assert bool((self.raw[-GUARD:] == PATTERN).all()), f"{name}: write after the buffer"
        assert bool(torch.isfinite(self.t.float()).all()), f"{name}: elements left unwritten"


@pytest.mark.parametrize("shape", [(1, 333, 12, 4, 16), (2, 129, 16, 1, 32), (1, 200, 6, 2, 64),
                                   (1, 257, 8, 4, 128)], ids=lambda s: "x".join(map(str, s)))
def test_fwd_bwd_write_only_their_outputs(cuda_lib, shape):
    B, N, Hq, Hkv, dh = shape
    q, k, v, dout = (t.cuda() for t in make_inputs(B, N, Hq, Hkv, dh, seed=2, with_dout=True))
    out, lse = Guarded((B, N, Hq, dh), torch.bfloat16), Guarded((B, Hq, N), torch.float32)
    cuda_lib.sqa_fwd(q, k, v, out=out.t, lse=lse.t, causal=True)
    out.check("out")
    lse.check("lse")
    dq, dk, dv = (Guarded(tuple(t.shape), torch.bfloat16) for t in (q, k, v))
    nbytes = cuda_lib.bwd_workspace_bytes(B, N, Hq, Hkv, dh)
    ws = Guarded((nbytes,), torch.uint8)
    ws.t.fill_(0)
    cuda_lib.sqa_bwd(dout, q, k, v, out.t, lse.t, dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t, causal=True)
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        g.check(name)
    torch.cuda.synchronize()
    assert bool((ws.raw[:GUARD] == PATTERN).all()) and bool((ws.raw[-GUARD:] == PATTERN).all()), "workspace"
    assert cuda_lib.device_status() == 0


@pytest.mark.parametrize("shape", [(1, 1500, 6, 1, 16), (1, 2500, 3, 1, 64)], ids=lambda s: "x".join(map(str, s)))
def test_fwd_key_ranges_write_only_their_outputs_and_workspace(cuda_lib, shape):
    """The key-range forward (partials, counters) stays inside its workspace."""
    B, N, Hq, Hkv, dh = shape
    nbytes = cuda_lib.fwd_workspace_bytes(B, N, Hq, Hkv, dh, True)
    assert nbytes > 0
    q, k, v, _ = (t.cuda() if t is not None else None for t in make_inputs(B, N, Hq, Hkv, dh, seed=4))
    out, lse = Guarded((B, N, Hq, dh), torch.bfloat16), Guarded((B, Hq, N), torch.float32)
    ws = Guarded((nbytes,), torch.uint8)
    cuda_lib.sqa_fwd(q, k, v, out=out.t, lse=lse.t, causal=True, workspace=ws.t)
    out.check("out")
    lse.check("lse")
    assert bool((ws.raw[:GUARD] == PATTERN).all()) and bool((ws.raw[-GUARD:] == PATTERN).all()), "workspace"
    assert cuda_lib.device_status() == 0


def test_decode_writes_only_its_outputs(cuda_lib):
    B, N, Hq, Hkv, dh = 3, 1000, 16, 1, 16
    q, k, v = (t.cuda() for t in make_decode_inputs(B, N, Hq, Hkv, dh, seed=3))
    lens = torch.tensor([1000, 77, 1], dtype=torch.int32, device="cuda")
    out, lse = Guarded((B, Hq, dh), torch.bfloat16), Guarded((B, Hq), torch.float32)
    nbytes = cuda_lib.decode_workspace_bytes(B, N, Hq, Hkv, dh)
    ws = Guarded((nbytes,), torch.uint8)
    cuda_lib.sqa_decode(q, k, v, seq_lens=lens, out=out.t, lse=lse.t, workspace=ws.t)
    out.check("decode out")
    lse.check("decode lse")
    assert bool((ws.raw[:GUARD] == PATTERN).all()) and bool((ws.raw[-GUARD:] == PATTERN).all()), "workspace"


def test_layer_writes_only_its_outputs(cuda_lib):
    B, N, d, Hq, Hkv, dh = 1, 333, 256, 8, 4, 16
    x, w_qkv, w_o, dy = (t.cuda() for t in make_layer_inputs(B, N, d, Hq, Hkv, dh, seed=4))
    y, saved = cuda_lib.sqa_layer_fwd(x, w_qkv, w_o, Hq, Hkv)
    lib = cuda_lib.load_library()
    s = cuda_lib.LayerShape(B, N, d, Hq, Hkv, dh)
    dx = Guarded((B, N, d), torch.bfloat16)
    dwq = Guarded(tuple(w_qkv.shape), torch.float32)
    dwo = Guarded(tuple(w_o.shape), torch.float32)
    nbytes = lib.sqa_layer_workspace_bytes(s, 1)
    ws = Guarded((nbytes,), torch.uint8)
    sv = saved
    st = lib.sqa_layer_bwd(dy.data_ptr(), x.data_ptr(), w_qkv.data_ptr(), w_o.data_ptr(), sv["q"].data_ptr(),
                           sv["k"].data_ptr(), sv["v"].data_ptr(), sv["out"].data_ptr(), sv["lse"].data_ptr(),
                           dx.t.data_ptr(), dwq.t.data_ptr(), dwo.t.data_ptr(), ws.t.data_ptr(), nbytes, s, 1,
                           ctypes.c_float(0.0), ctypes.c_float(10000.0),
                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.sqa_last_error()
    for name, g in (("dx", dx), ("dw_qkv", dwq), ("dw_o", dwo)):
        g.check(name)
    assert bool((ws.raw[:GUARD] == PATTERN).all()) and bool((ws.raw[-GUARD:] == PATTERN).all()), "workspace"
    assert cuda_lib.device_status() == 0
