"""GPU parity of sqa_decode (one new token per sequence against its key/value
cache) with the fp64 oracle, on seeded inputs; ragged cache lengths, group
sizes 1-128, every head dim, K/V head counts that are and are not powers of
two (the register-resident split path takes groups of at most four heads with a
power-of-two K/V head count, the tensor-core path groups of 5 to 16 heads, the
shared-memory path the rest), a one-entry
cache, the whole cache, an empty sequence, and the full-size decoding
workloads."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, assert_lse_close, to_np
from sparse_query_attention_sqa_b200.inputs import WORKLOADS, make_decode_inputs

pytestmark = pytest.mark.gpu


def _inputs(B, N, Hq, Hkv, dh, seed, k_scale=1.0, std=1.0):
    return make_decode_inputs(B, N, Hq, Hkv, dh, seed=seed, k_scale=k_scale, std=std)


def _run(cuda_lib, q, k, v, lens):
    lens_d = None if lens is None else torch.tensor(lens, dtype=torch.int32).cuda()
    out, lse = cuda_lib.sqa_decode(q.cuda(), k.cuda(), v.cuda(), seq_lens=lens_d)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    return to_np(out), lse.cpu().numpy().astype(np.float64)


CASES = [
    ((3, 300, 8, 4, 16), [1, 128, 300]),
    ((2, 1000, 16, 1, 16), [999, 257]),
    ((2, 129, 4, 4, 128), None),
    ((1, 4096, 8, 2, 32), None),
    ((4, 700, 12, 4, 64), [700, 129, 128, 5]),
    ((2, 1, 8, 4, 16), None),
    ((2, 3000, 128, 1, 16), [2999, 3]),
    ((2, 520, 16, 2, 128), [520, 131]),
    ((1, 400, 32, 8, 64), None),
    ((2, 300, 16, 16, 128), [300, 17]),
    ((2, 500, 6, 3, 32), [500, 250]),
    ((1, 5000, 8, 2, 128), [4999]),
    # groups of 5 to 16 heads: the tensor-core split path
    ((2, 777, 10, 2, 64), [777, 300]),
    ((3, 1500, 36, 3, 32), [1500, 1, 1025]),
    ((2, 2049, 16, 1, 128), [2049, 64]),
    ((1, 200, 7, 1, 16), None),
    ((2, 130, 40, 4, 128), [1, 130]),
]


@pytest.mark.parametrize("shape,lens", CASES, ids=lambda c: "x".join(map(str, c)) if isinstance(c, tuple) else str(c))
def test_decode_matches_oracle(cuda_lib, shape, lens):
    q, k, v = _inputs(*shape, seed=7)
    out, lse = _run(cuda_lib, q, k, v, lens)
    ref_out, ref_lse = oracle.sqa_decode(q, k, v, lens)
    assert_lse_close("lse", lse, ref_lse)
    assert_close("out", out, ref_out)


def test_zero_query_averages_the_prefix(cuda_lib):
    _, k, v = _inputs(2, 600, 8, 4, 16, seed=3)
    q = torch.zeros(2, 8, 16, dtype=torch.bfloat16)
    out, lse = _run(cuda_lib, q, k, v, [600, 77])
    ref_out, ref_lse = oracle.sqa_decode(q, k, v, [600, 77])
    assert_close("out", out, ref_out)
    np.testing.assert_allclose(lse, np.log(np.array([[600.0] * 8, [77.0] * 8])), atol=1e-4)


def test_empty_sequence_gives_zero_output(cuda_lib):
    q, k, v = _inputs(2, 300, 8, 4, 16, seed=4)
    out, lse = _run(cuda_lib, q, k, v, [0, 300])
    assert np.all(out[0] == 0.0) and np.all(np.isneginf(lse[0]))
    ref_out, ref_lse = oracle.sqa_decode(q[1:], k[1:], v[1:], [300])
    assert_close("out", out[1:], ref_out)
    assert_lse_close("lse", lse[1:], ref_lse)


def test_cache_past_the_length_is_not_read(cuda_lib):
    q, k, v = _inputs(1, 1000, 8, 4, 16, seed=5)
    a = _run(cuda_lib, q, k, v, [300])
    k2, v2 = k.clone(), v.clone()
    k2[:, 300:] = float("nan")
    v2[:, 300:] = float("inf")
    b = _run(cuda_lib, q, k2, v2, [300])
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("Hq,Hkv,dh", [(10, 1, 16), (16, 2, 128)])
def test_tensor_core_path_ignores_the_cache_past_the_length(cuda_lib, Hq, Hkv, dh):
    q, k, v = _inputs(1, 1500, Hq, Hkv, dh, seed=8)
    a = _run(cuda_lib, q, k, v, [1100])
    k2, v2 = k.clone(), v.clone()
    k2[:, 1100:] = float("nan")
    v2[:, 1100:] = float("inf")
    b = _run(cuda_lib, q, k2, v2, [1100])
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("Hq,Hkv,dh", [(10, 1, 16), (12, 2, 64), (16, 2, 128), (5, 1, 32)])
def test_growing_scores_raise_the_running_maximum(cuda_lib, Hq, Hkv, dh):
    # keys scaled up along the cache: later positions raise the running maximum
    # by more than the kernels' lazy-rescale threshold, inside and across ranges
    q, k, v = _inputs(2, 3000, Hq, Hkv, dh, seed=9)
    ramp = (1.0 + torch.arange(3000, dtype=torch.float32) / 300.0).to(torch.bfloat16)
    k = (k.float() * ramp[None, :, None, None].float()).to(torch.bfloat16)
    out, lse = _run(cuda_lib, q, k, v, [3000, 1777])
    ref_out, ref_lse = oracle.sqa_decode(q, k, v, [3000, 1777])
    assert_lse_close("lse", lse, ref_lse)
    assert_close("out", out, ref_out)


def test_workspace_contents_do_not_matter(cuda_lib):
    B, N, Hq, Hkv, dh = 2, 900, 8, 4, 32
    q, k, v = _inputs(B, N, Hq, Hkv, dh, seed=6)
    ws = torch.full((cuda_lib.decode_workspace_bytes(B, N, Hq, Hkv, dh),), 0x7F, dtype=torch.uint8).cuda()
    out, lse = cuda_lib.sqa_decode(q.cuda(), k.cuda(), v.cuda(), workspace=ws)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.sqa_decode(q, k, v)
    assert_close("out", to_np(out), ref_out)
    assert_lse_close("lse", lse.cpu().numpy(), ref_lse)


@pytest.mark.parametrize("name", ["decode_sqatm", "decode_dh128", "decode_mqa"])
def test_decode_workloads_full_size(cuda_lib, name):
    w = WORKLOADS[name]
    q, k, v = _inputs(w.B, w.N, w.Hq, w.Hkv, w.dh, seed=0, k_scale=w.k_scale, std=w.std)
    out, lse = _run(cuda_lib, q, k, v, None)
    ref_out, ref_lse = oracle.sqa_decode(q, k, v, None, w.scale)
    assert_lse_close("lse", lse, ref_lse)
    assert_close("out", out, ref_out)
