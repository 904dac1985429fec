"""GPU parity of the full SQA layer (sqa_layer_fwd / sqa_layer_bwd: fused Q/K/V
projection with the rotary embedding in its epilogue, the attention core, the
output projection, and the backward with the weight gradients) against the
fp64 oracle of ``oracle/layer.py``.

Tolerance.  The layer stores its intermediates as the core takes and gives
them, in bf16: the rotated q, k, v, the core output, dO and the core's dq, dk,
dv (then dq, dk rotated back and rounded again).  Each rounding is up to half a
bf16 ulp (relative 2^-9), and the oracle rounds nothing.  Replaying the oracle
with exactly those roundings and nothing else gives relative Frobenius errors
of 3.0e-3 to 4.7e-3 and largest errors of 0.015 to 0.065 times the RMS of the
exact result, over the shapes below.  The bar is therefore relative Frobenius
<= 1e-2 and, element by element, |error| <= 2e-2 + 0.1 * RMS(exact).
"""
import numpy as np
import pytest
import torch

from oracle.layer import sqa_layer_bwd, sqa_layer_fwd
from parity import assert_scaled_close as assert_layer_close, to_np
from sparse_query_attention_sqa_b200.inputs import make_layer_inputs

pytestmark = pytest.mark.gpu

# (B, N, d, H_q, H_kv, dh, causal): the SQAT-m layer (d = 256 over 16 heads,
# 8 query heads, 4 key/value heads), a ragged token count (M not a multiple of
# the 128-row tile), MQA and MHA head layouts, and a dh = 128 model.
SHAPES = [
    (2, 256, 256, 8, 4, 16, True),
    (3, 200, 256, 8, 4, 16, False),
    (1, 300, 256, 16, 1, 16, True),
    (1, 128, 256, 16, 16, 16, True),
    (1, 256, 1024, 8, 4, 128, True),
]


def run_layer(cuda_lib, B, N, d, Hq, Hkv, dh, causal, rope_base=10000.0, seed=0):
    x, w_qkv, w_o, dy = make_layer_inputs(B, N, d, Hq, Hkv, dh, seed=seed)
    xd, wd, wod, dyd = (t.cuda() for t in (x, w_qkv, w_o, dy))
    y, saved = cuda_lib.sqa_layer_fwd(xd, wd, wod, Hq, Hkv, causal=causal, rope_base=rope_base)
    dx, dw_qkv, dw_o = cuda_lib.sqa_layer_bwd(dyd, xd, wd, wod, saved, Hq, Hkv, causal=causal, rope_base=rope_base)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    nq, nk = Hq * dh, Hkv * dh
    xf, wf, wof, dyf = (t.double().numpy() for t in (x, w_qkv, w_o, dy))
    wq, wk, wv = wf[:, :nq], wf[:, nq:nq + nk], wf[:, nq + nk:]
    base = rope_base if rope_base > 0 else None
    ref_y, mid = sqa_layer_fwd(xf, wq, wk, wv, wof, Hq, Hkv, causal, rope_base=base)
    rdx, rdwq, rdwk, rdwv, rdwo = sqa_layer_bwd(xf, wq, wk, wv, wof, dyf, Hq, Hkv, causal, rope_base=base)
    got = {"y": to_np(y), "q": to_np(saved["q"]), "k": to_np(saved["k"]), "v": to_np(saved["v"]), "dx": to_np(dx),
           "dw_qkv": to_np(dw_qkv), "dw_o": to_np(dw_o)}
    ref = {"y": ref_y, "q": mid["q"], "k": mid["k"], "v": mid["v"], "dx": rdx,
           "dw_qkv": np.concatenate([rdwq, rdwk, rdwv], axis=1), "dw_o": rdwo}
    return got, ref


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_layer_matches_oracle(cuda_lib, shape):
    got, ref = run_layer(cuda_lib, *shape)
    for name in ("q", "k", "v", "y", "dx", "dw_qkv", "dw_o"):
        assert_layer_close(name, got[name], ref[name])


def test_layer_without_rotation(cuda_lib):
    """rope_base = 0 leaves Q and K as projected."""
    got, ref = run_layer(cuda_lib, 1, 200, 256, 8, 4, 16, True, rope_base=0.0)
    for name in ("q", "k", "y", "dx", "dw_qkv"):
        assert_layer_close(name, got[name], ref[name])


def test_layer_projections_are_exact_products(cuda_lib):
    """The projection GEMM alone, checked tightly: q, k, v are each one bf16
    rounding of an fp32-accumulated product of bf16 values (q and k turned by
    fp32 cos/sin first), so they must lie within half a bf16 ulp (plus the
    fp32 arithmetic) of the exact result."""
    from parity import bf16_half_ulp

    B, N, d, Hq, Hkv, dh = 1, 333, 256, 8, 4, 16
    got, ref = run_layer(cuda_lib, B, N, d, Hq, Hkv, dh, True)
    for name in ("q", "k", "v"):
        err = np.abs(got[name] - ref[name])
        assert np.all(err <= bf16_half_ulp(ref[name]) + 1e-5 * (1 + np.abs(ref[name]))), name
