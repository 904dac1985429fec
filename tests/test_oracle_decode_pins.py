"""Pins of the oracle's decoding step (one new token per sequence against its
key/value cache), CPU only.

Each test fixes the result by something other than the oracle itself: an
independent per-head numpy computation, closed forms (a one-entry cache, an
all-zero query), invariances (entries past the length, joint permutation of
the cache rows), and agreement with the last row of the full causal forward.
"""
import numpy as np
import pytest

import oracle


def _brute(q, k, v, lens, scale):
    B, Hq, dh = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    out = np.zeros((B, Hq, dh))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            kk = k[b, : lens[b], h // g]
            vv = v[b, : lens[b], h // g]
            s = scale * (kk @ q[b, h])
            m = s.max()
            w = np.exp(s - m)
            lse[b, h] = m + np.log(w.sum())
            out[b, h] = (w / w.sum()) @ vv
    return out, lse


@pytest.mark.parametrize("Hq,Hkv,dh", [(8, 4, 16), (16, 1, 16), (4, 4, 128), (12, 4, 32)])
def test_matches_independent_brute_force(Hq, Hkv, dh):
    rng = np.random.default_rng(Hq * 100 + dh)
    B, N = 3, 37
    q = rng.standard_normal((B, Hq, dh))
    k = rng.standard_normal((B, N, Hkv, dh))
    v = rng.standard_normal((B, N, Hkv, dh))
    lens = np.array([1, 20, 37])
    scale = 1.0 / np.sqrt(dh)
    out, lse = oracle.sqa_decode(q, k, v, lens)
    ref_out, ref_lse = _brute(q, k, v, lens, scale)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_one_entry_cache_returns_that_value():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 8, 16))
    k = rng.standard_normal((2, 5, 4, 16))
    v = rng.standard_normal((2, 5, 4, 16))
    out, lse = oracle.sqa_decode(q, k, v, [1, 1], scale=0.25)
    for h in range(8):
        np.testing.assert_array_equal(out[:, h], v[:, 0, h // 2])
        np.testing.assert_allclose(lse[:, h], 0.25 * np.einsum("bd,bd->b", q[:, h], k[:, 0, h // 2]), atol=1e-14)


def test_zero_query_averages_the_prefix():
    rng = np.random.default_rng(2)
    k = rng.standard_normal((2, 9, 2, 16))
    v = rng.standard_normal((2, 9, 2, 16))
    lens = np.array([4, 9])
    out, lse = oracle.sqa_decode(np.zeros((2, 6, 16)), k, v, lens)
    for b in range(2):
        for h in range(6):
            np.testing.assert_allclose(out[b, h], v[b, : lens[b], h // 3].mean(axis=0), atol=1e-14)
            assert lse[b, h] == pytest.approx(np.log(lens[b]), abs=1e-14)


def test_cache_entries_past_the_length_do_not_matter():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((2, 4, 32))
    k = rng.standard_normal((2, 12, 2, 32))
    v = rng.standard_normal((2, 12, 2, 32))
    lens = np.array([5, 8])
    a = oracle.sqa_decode(q, k, v, lens)
    k2, v2 = k.copy(), v.copy()
    k2[0, 5:] = 1e3
    v2[1, 8:] = -7.0
    b = oracle.sqa_decode(q, k2, v2, lens)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_joint_permutation_of_cache_rows():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 8, 16))
    k = rng.standard_normal((1, 20, 4, 16))
    v = rng.standard_normal((1, 20, 4, 16))
    perm = rng.permutation(20)
    a = oracle.sqa_decode(q, k, v)
    b = oracle.sqa_decode(q, k[:, perm], v[:, perm])
    np.testing.assert_allclose(a[0], b[0], atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], atol=1e-12)


def test_equals_last_row_of_the_causal_forward():
    rng = np.random.default_rng(5)
    B, N, Hq, Hkv, dh = 2, 30, 8, 2, 16
    q = rng.standard_normal((B, N, Hq, dh))
    k = rng.standard_normal((B, N, Hkv, dh))
    v = rng.standard_normal((B, N, Hkv, dh))
    out, lse = oracle.sqa_fwd(q, k, v, causal=True)
    dout, dlse = oracle.sqa_decode(q[:, -1], k, v)
    np.testing.assert_allclose(dout, out[:, -1], atol=1e-12)
    np.testing.assert_allclose(dlse, lse[:, :, -1], atol=1e-12)


@pytest.mark.parametrize("lens", [[0, 3], [3, 6]])
def test_rejects_lengths_outside_the_cache(lens):
    q = np.zeros((2, 4, 16))
    k = np.zeros((2, 5, 2, 16))
    with pytest.raises(ValueError):
        oracle.sqa_decode(q, k, k, lens)
