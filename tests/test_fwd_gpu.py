"""GPU parity of sqa_fwd against the fp64 oracle, element by element."""
import numpy as np
import pytest
import torch

import oracle
from sparse_query_attention_sqa_b200.inputs import make_inputs
from parity import assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu

# (B, N, H_q, H_kv, dh): several 128-row tiles, ragged tails, and every
# group-size class (g = 1 MHA, 2, 3 and 6 which do not divide 128, 4, 16 MQA).
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
    # more work items than SMs, so every persistent CTA walks several items
    # (buffer and barrier phases carried across items), with ragged tails
    (6, 1000, 8, 4, 16),
    (26, 300, 8, 2, 32),
    (4, 1216, 8, 4, 128),  # 160 forward items of 148 SMs: turns in CTAs that walk several items, one-tile items
]


def run(cuda_lib, B, N, Hq, Hkv, dh, causal, seed=0, std=1.0, k_scale=1.0, scale=0.0):
    q, k, v, _ = make_inputs(B, N, Hq, Hkv, dh, seed=seed, std=std, k_scale=k_scale)
    out, lse = cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    ref_out, ref_lse = oracle.sqa_fwd(q, k, v, causal, scale if scale > 0 else None)
    return to_np(out), to_np(lse), ref_out, ref_lse


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fwd_matches_oracle(cuda_lib, shape, causal):
    out, lse, ref_out, ref_lse = run(cuda_lib, *shape, causal)
    # lse alone checks the QK^T contraction and the softmax statistics;
    # O additionally checks the PV contraction.
    assert_lse_close("lse", lse, ref_lse)
    assert_close("out", out, ref_out)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_zero_query_gives_prefix_mean(cuda_lib, causal):
    """All-zero Q exercises the PV contraction independently of QK^T."""
    B, N, Hq, Hkv, dh = 1, 300, 8, 4, 16
    _, k, v, _ = make_inputs(B, N, Hq, Hkv, dh, seed=3)
    q = torch.zeros(B, N, Hq, dh, dtype=torch.bfloat16)
    out, lse = cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal)
    ref_out, ref_lse = oracle.sqa_fwd(q, k, v, causal)
    assert_lse_close("lse", to_np(lse), ref_lse)
    assert_close("out", to_np(out), ref_out)


def test_explicit_scale_and_seeds(cuda_lib):
    for seed in (1, 2):
        out, lse, ref_out, ref_lse = run(cuda_lib, 2, 300, 8, 4, 16, True, seed=seed, scale=0.25)
        assert_lse_close("lse", lse, ref_lse)
        assert_close("out", out, ref_out)


@pytest.mark.parametrize("std,scale", [(2.0, 1.0), (1.0, 3.0)], ids=["std2_scale1", "std1_scale3"])
def test_wide_score_range_rescales_exactly(cuda_lib, std, scale):
    """Large scores force the running maximum up many times along a row: with
    Q, K and V of standard deviation 2 and scale 1 the scores have standard
    deviation 16 (each row is close to one-hot and |O| reaches about 8); with
    unit inputs and scale 3, 12."""
    out, lse, ref_out, ref_lse = run(cuda_lib, 1, 700, 8, 4, 16, False, std=std, scale=scale)
    assert_lse_close("lse", lse, ref_lse)
    assert_close("out", out, ref_out)


def test_outputs_fully_overwritten_and_inputs_untouched(cuda_lib):
    B, N, Hq, Hkv, dh = 1, 200, 8, 4, 16
    q, k, v, _ = make_inputs(B, N, Hq, Hkv, dh, seed=4)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out = torch.full((B, N, Hq, dh), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device="cuda")
    cuda_lib.sqa_fwd(qd, kd, vd, out=out, lse=lse, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    assert torch.equal(qd.cpu(), q) and torch.equal(kd.cpu(), k) and torch.equal(vd.cpu(), v)


def test_deterministic(cuda_lib):
    q, k, v, _ = make_inputs(2, 333, 8, 4, 16, seed=5)
    a = cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    b = cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_errors_launch_nothing(cuda_lib):
    from sparse_query_attention_sqa_b200 import SqaError

    q, k, v, _ = make_inputs(1, 64, 6, 4, 16)
    with pytest.raises(SqaError) as e:
        cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda())
    assert e.value.status == 1
    q, k, v, _ = make_inputs(1, 64, 4, 4, 48)
    with pytest.raises(SqaError) as e:
        cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda())
    assert e.value.status == 2


# Small problems whose Q tiles fill less than half the SMs: the key tiles of
# each Q tile are split into ranges computed by separate CTAs and merged by the
# last range to finish (sqa_fwd_with_workspace).  g = 3 and g = 6 leave rows
# with no visible key in a later range (tokens of a tile before that range's
# first key).
RANGE_SHAPES = [
    (1, 2000, 2, 1, 32),  # eight ranges per Q tile at the end of the causal sequence
    (1, 4096, 2, 1, 16),  # 148 items of up to 18 key tiles
    (1, 2500, 3, 1, 64),
    (1, 1500, 6, 1, 16),
    (2, 1500, 2, 1, 32),
    (1, 1000, 2, 2, 16),  # MHA layout: 128 tokens per Q tile
]


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", RANGE_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fwd_key_ranges_match_oracle_and_one_cta_per_tile(cuda_lib, shape, causal):
    """The ranges path (workspace filled with 0xff bytes first: the call clears
    its counters itself) and the one-CTA-per-Q-tile path both match the oracle;
    a second call with the same workspace gives the same bits."""
    assert cuda_lib.fwd_workspace_bytes(*shape, causal) > 0, "shape does not take the ranges path"
    q, k, v, _ = make_inputs(*shape, seed=6)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    ws = torch.full((cuda_lib.fwd_workspace_bytes(*shape, causal),), 255, dtype=torch.uint8, device="cuda")
    out_r, lse_r = cuda_lib.sqa_fwd(qd, kd, vd, causal=causal, workspace=ws)
    out_r2, lse_r2 = cuda_lib.sqa_fwd(qd, kd, vd, causal=causal, workspace=ws)
    out_1, lse_1 = cuda_lib.sqa_fwd(qd, kd, vd, causal=causal, key_ranges=False)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    ref_out, ref_lse = oracle.sqa_fwd(q, k, v, causal, None)
    for out, lse in ((out_r, lse_r), (out_1, lse_1)):
        assert_lse_close("lse", to_np(lse), ref_lse)
        assert_close("out", to_np(out), ref_out)
    assert torch.equal(out_r, out_r2) and torch.equal(lse_r, lse_r2)
