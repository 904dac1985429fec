"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times.

The oracle cannot run every output at these sizes in seconds, so each test
checks outputs it can compute one by one: whole batch entries (batch entries
are independent problems) or sampled query rows including row 0, the last row
and rows of the ragged last tile, and for the dh = 128 backward the last key
rows, whose gradients only involve the last query rows under the causal mask.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_query_attention_sqa_b200.inputs import WORKLOADS, workload_inputs
from parity import assert_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu


def sample_rows(N, n, rng, tail=128):
    rows = {0, N - 1, N // 2}
    rows.update(range(max(0, N - tail), N, max(1, tail // 16)))  # ragged last tile
    rows.update(int(i) for i in rng.integers(0, N, n))
    return np.array(sorted(rows))


def test_sqatm_layer_fwd_full(cuda_lib):
    w = WORKLOADS["sqatm_layer_fwd"]
    q, k, v, _ = workload_inputs(w)
    out, lse = cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, scale=w.scale)
    ref_out, ref_lse = oracle.sqa_fwd(q, k, v, w.causal, w.softmax_scale)
    assert_lse_close("lse", to_np(lse), ref_lse)
    assert_close("out", to_np(out), ref_out)


@pytest.mark.parametrize("name", ["sqatm_train_sqa", "sqatm_train_gqa", "sqatm_train_mha", "sqatm_train_mqa"])
def test_sqatm_train_fwd_bwd_batches(cuda_lib, name):
    """Full B=32 launch; batch entries 0, 17 and 31 checked completely."""
    w = WORKLOADS[name]
    q, k, v, dout = workload_inputs(w)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = cuda_lib.sqa_fwd(qd, kd, vd, causal=w.causal)
    dq, dk, dv = cuda_lib.sqa_bwd(dod, qd, kd, vd, out, lse, causal=w.causal)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    for b in (0, 17, 31):
        sl = slice(b, b + 1)
        ref_out, ref_lse = oracle.sqa_fwd(q[sl], k[sl], v[sl], w.causal)
        assert_lse_close(f"lse[b={b}]", to_np(lse[sl]), ref_lse)
        assert_close(f"out[b={b}]", to_np(out[sl]), ref_out)
        rdq, rdk, rdv = oracle.sqa_bwd(q[sl], k[sl], v[sl], dout[sl], w.causal)
        assert_close(f"dv[b={b}]", to_np(dv[sl]), rdv)
        assert_close(f"dk[b={b}]", to_np(dk[sl]), rdk)
        assert_close(f"dq[b={b}]", to_np(dq[sl]), rdq)


ENCODER = [n for n in WORKLOADS if n.startswith("enc")]


@pytest.mark.parametrize("name", ENCODER)
def test_long_encoder_fwd_sampled_rows(cuda_lib, name):
    w = WORKLOADS[name]
    q, k, v, _ = workload_inputs(w)
    out, lse = cuda_lib.sqa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=w.causal)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    rng = np.random.default_rng(0)
    per_head = 24 if w.N > 100000 else 48
    rows = sample_rows(w.N, per_head, rng)
    trip = np.array([(0, i, h) for h in range(w.Hq) for i in rows])
    ref_o, ref_l = oracle.sqa_fwd_rows(q, k, v, trip, w.causal)
    o = to_np(out)[0][trip[:, 1], trip[:, 2]]
    l = to_np(lse)[0][trip[:, 2], trip[:, 1]]
    assert_lse_close("lse", l, ref_l)
    assert_close("out", o, ref_o)


def test_large_dh128_fwd_bwd_sampled(cuda_lib):
    w = WORKLOADS["large_dh128"]
    q, k, v, dout = workload_inputs(w)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = cuda_lib.sqa_fwd(qd, kd, vd, causal=w.causal)
    dq, dk, dv = cuda_lib.sqa_bwd(dod, qd, kd, vd, out, lse, causal=w.causal)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    # batch entry 1 only, so the fp64 copies stay small
    q1, k1, v1, do1 = q[1:2], k[1:2], v[1:2], dout[1:2]
    rng = np.random.default_rng(1)
    rows = sample_rows(w.N, 6, rng, tail=64)
    qtrip = np.array([(0, i, h) for h in range(w.Hq) for i in rows])
    ref_o, ref_l = oracle.sqa_fwd_rows(q1, k1, v1, qtrip, w.causal)
    assert_lse_close("lse", to_np(lse[1])[qtrip[:, 2], qtrip[:, 1]], ref_l)
    assert_close("out", to_np(out[1])[qtrip[:, 1], qtrip[:, 2]], ref_o)
    drows = np.array([0, 1, 777, w.N // 2, w.N - 2, w.N - 1])
    dtrip = np.array([(0, i, h) for h in range(w.Hq) for i in drows])
    ktrip = np.array([(0, j, kv) for kv in range(w.Hkv) for j in range(w.N - 48, w.N)])
    rdq, rdk, rdv = oracle.sqa_bwd_rows(q1, k1, v1, do1, dtrip, ktrip, w.causal)
    assert_close("dq", to_np(dq[1])[dtrip[:, 1], dtrip[:, 2]], rdq)
    assert_close("dk", to_np(dk[1])[ktrip[:, 1], ktrip[:, 2]], rdk)
    assert_close("dv", to_np(dv[1])[ktrip[:, 1], ktrip[:, 2]], rdv)


def test_dh128_full_check_small(cuda_lib):
    """Every output of a 1536-token problem with the dh = 128 head shape."""
    from sparse_query_attention_sqa_b200.inputs import make_inputs

    q, k, v, dout = make_inputs(1, 1536, 8, 4, 128, seed=3, k_scale=0.1, with_dout=True)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = cuda_lib.sqa_fwd(qd, kd, vd, causal=True)
    dq, dk, dv = cuda_lib.sqa_bwd(dod, qd, kd, vd, out, lse, causal=True)
    ref_out, ref_lse = oracle.sqa_fwd(q, k, v, True)
    assert_lse_close("lse", to_np(lse), ref_lse)
    assert_close("out", to_np(out), ref_out)
    rdq, rdk, rdv = oracle.sqa_bwd(q, k, v, dout, True)
    assert_close("dv", to_np(dv), rdv)
    assert_close("dk", to_np(dk), rdk)
    assert_close("dq", to_np(dq), rdq)
