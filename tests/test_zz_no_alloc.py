"""sqa_bwd_static_scratch: the backward for callers that cannot allocate device
memory (for example a plugin inside a framework that owns every device
allocation).  It must give the same gradients as sqa_bwd with a caller-owned
workspace, on consecutive calls that reuse its one static scratch array.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from sparse_query_attention_sqa_b200.inputs import make_inputs
from parity import assert_close, to_np

pytestmark = pytest.mark.gpu


def _entry(lib):
    f = lib.sqa_bwd_static_scratch
    vp = ctypes.c_void_p
    import sparse_query_attention_sqa_b200 as sqa

    f.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, sqa.Shape, ctypes.c_int, ctypes.c_float, vp]
    f.restype = ctypes.c_int
    return f


@pytest.mark.parametrize("shape,causal", [((2, 300, 8, 4, 16), True), ((1, 257, 16, 1, 16), False),
                                          ((1, 200, 8, 4, 128), True)])
def test_static_scratch_backward_matches_workspace_backward(cuda_lib, shape, causal):
    B, N, Hq, Hkv, dh = shape
    lib = cuda_lib.load_library()
    entry = _entry(lib)
    q, k, v, dout = (t.cuda() for t in make_inputs(B, N, Hq, Hkv, dh, seed=11, with_dout=True))
    out, lse = cuda_lib.sqa_fwd(q, k, v, causal=causal)
    ref = cuda_lib.sqa_bwd(dout, q, k, v, out, lse, causal=causal)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):  # the second call reuses the scratch the first one left behind
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        st = entry(dout.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                   dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cuda_lib.Shape(B, N, Hq, Hkv, dh), int(causal),
                   ctypes.c_float(0.0), stream)
        assert st == 0, lib.sqa_last_error()
        torch.cuda.synchronize()
        assert cuda_lib.device_status() == 0
        for name, got, want in (("dq", dq, ref[0]), ("dk", dk, ref[1]), ("dv", dv, ref[2])):
            assert_close(name, to_np(got), to_np(want))


def test_static_scratch_rejects_shapes_beyond_its_size(cuda_lib):
    lib = cuda_lib.load_library()
    entry = _entry(lib)
    s = cuda_lib.Shape(4, 65536, 16, 4, 16)
    lib.sqa_bwd_workspace_bytes.restype = ctypes.c_size_t
    assert lib.sqa_bwd_workspace_bytes(s) > 64 * 1024 * 1024  # this shape needs more than the static scratch
    # Null tensors: whatever the checks' order, nothing can be launched.
    st = entry(*([None] * 9), s, 1, ctypes.c_float(0.0), None)
    assert st == 2
    assert b"static scratch" in lib.sqa_last_error()
