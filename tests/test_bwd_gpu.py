"""GPU parity of sqa_bwd against the fp64 oracle, element by element."""
import pytest
import torch

import oracle
from sparse_query_attention_sqa_b200.inputs import make_inputs
from parity import assert_close, to_np

pytestmark = pytest.mark.gpu

SHAPES = [
    (1, 1, 8, 4, 16),
    (1, 7, 8, 4, 16),
    (2, 300, 8, 4, 16),
    (1, 1024, 8, 4, 16),
    (2, 257, 16, 16, 16),
    (2, 200, 16, 1, 16),
    (1, 333, 12, 4, 16),
    (1, 513, 6, 1, 16),
    (2, 129, 16, 4, 16),
    (1, 390, 8, 4, 32),
    (1, 390, 8, 4, 64),
    (2, 300, 8, 4, 128),
    (1, 129, 4, 4, 128),
    (1, 200, 16, 1, 128),  # MQA at dh 128: 8 tokens per Q tile
    (2, 150, 12, 4, 128),  # g = 3: 126 of the 128 tile rows used
    (1, 257, 12, 2, 64),
    (1, 300, 8, 1, 64),    # g = 8: dK/dV take P and dS as two bf16 terms
    (2, 200, 14, 2, 64),   # g = 7: likewise (0.020 of dV error with one term)
    (1, 300, 5, 1, 64),    # g = 5: the largest group that takes them as one
    # more work items than SMs, so every persistent CTA walks several items
    # (buffer and barrier phases carried across items), with ragged tails
    (6, 1000, 8, 4, 16),
    (26, 300, 8, 2, 32),
    (4, 1216, 8, 4, 128),  # 160 forward items of 148 SMs: turns in CTAs that walk several items, one-tile items
]


def run_bwd(cuda_lib, B, N, Hq, Hkv, dh, causal, seed=0, scale=0.0, k_scale=1.0):
    q, k, v, dout = make_inputs(B, N, Hq, Hkv, dh, seed=seed, k_scale=k_scale, with_dout=True)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = cuda_lib.sqa_fwd(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = cuda_lib.sqa_bwd(dod, qd, kd, vd, out, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    ref = oracle.sqa_bwd(q, k, v, dout, causal, scale if scale > 0 else None)
    return (to_np(dq), to_np(dk), to_np(dv)), ref


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_bwd_matches_oracle(cuda_lib, shape, causal):
    (dq, dk, dv), (rdq, rdk, rdv) = run_bwd(cuda_lib, *shape, causal)
    # dV depends only on P and dO; dK and dQ add dS.
    assert_close("dv", dv, rdv)
    assert_close("dk", dk, rdk)
    assert_close("dq", dq, rdq)


def test_bwd_explicit_scale_and_seeds(cuda_lib):
    for seed in (1, 2):
        (dq, dk, dv), (rdq, rdk, rdv) = run_bwd(cuda_lib, 2, 300, 8, 4, 16, True, seed=seed, scale=0.25)
        assert_close("dv", dv, rdv)
        assert_close("dk", dk, rdk)
        assert_close("dq", dq, rdq)


def test_bwd_workspace_contents_do_not_matter(cuda_lib):
    B, N, Hq, Hkv, dh = 1, 300, 8, 4, 16
    q, k, v, dout = make_inputs(B, N, Hq, Hkv, dh, seed=7, with_dout=True)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = cuda_lib.sqa_fwd(qd, kd, vd, causal=True)
    nbytes = cuda_lib.bwd_workspace_bytes(B, N, Hq, Hkv, dh)
    ws = torch.full((nbytes,), 0x7F, dtype=torch.uint8, device="cuda")
    a = cuda_lib.sqa_bwd(dod, qd, kd, vd, out, lse, workspace=ws, causal=True)
    ws.fill_(0xFF)
    b = cuda_lib.sqa_bwd(dod, qd, kd, vd, out, lse, workspace=ws, causal=True)
    torch.cuda.synchronize()
    # dK and dV are exact reruns; dQ sums atomics in a run-dependent order.
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() < 1e-2


def test_bwd_outputs_fully_overwritten(cuda_lib):
    B, N, Hq, Hkv, dh = 1, 200, 16, 4, 16
    q, k, v, dout = make_inputs(B, N, Hq, Hkv, dh, seed=8, with_dout=True)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = cuda_lib.sqa_fwd(qd, kd, vd, causal=False)
    nan = float("nan")
    dq = torch.full_like(qd, nan)
    dk = torch.full_like(kd, nan)
    dv = torch.full_like(vd, nan)
    cuda_lib.sqa_bwd(dod, qd, kd, vd, out, lse, dq=dq, dk=dk, dv=dv, causal=False)
    torch.cuda.synchronize()
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
