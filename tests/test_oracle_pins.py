"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: a per-head
numpy brute force written independently here, the MHA/MQA special cases of
grouped heads (GQA summary, "The notation": GQA-1 is MQA and GQA-H is MHA),
closed forms (all-zero Q gives uniform weights), symmetries (token permutation
equivariance), central finite differences of the forward for the backward, and
two conservation sums of the backward.  A plausible slip in the oracle (a
wrong group map, a dropped scale, a transposed operand, an off-by-one causal
mask, a missing term in dS) breaks at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from sparse_query_attention_sqa_b200.inputs import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def brute_mha(q, k, v, causal, scale):
    """Per-head softmax(Q K^T * scale) V with numpy matrices; q, k, v all [B,N,H,dh]."""
    B, N, H, dh = q.shape
    out = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            S = (q[b, :, h, :] @ k[b, :, h, :].T) * scale
            if causal:
                S[np.triu_indices(N, 1)] = -np.inf
            m = S.max(axis=1, keepdims=True)
            E = np.exp(S - m)
            Z = E.sum(axis=1, keepdims=True)
            out[b, :, h, :] = (E / Z) @ v[b, :, h, :]
            lse[b, h, :] = (m + np.log(Z))[:, 0]
    return out, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,dh", [(1, 16), (5, 16), (33, 16), (19, 128), (7, 32)])
def test_mha_matches_brute_force(causal, N, dh):
    q, k, v = rand((2, N, 3, dh), 1), rand((2, N, 3, dh), 2), rand((2, N, 3, dh), 3)
    scale = dh ** -0.5
    out, lse = oracle.sqa_fwd(q, k, v, causal, scale)
    ref_out, ref_lse = brute_mha(q, k, v, causal, scale)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_mqa_matches_broadcast_brute_force(causal):
    Hq, N, dh = 6, 23, 16
    q, k, v = rand((2, N, Hq, dh), 4), rand((2, N, 1, dh), 5), rand((2, N, 1, dh), 6)
    out, lse = oracle.sqa_fwd(q, k, v, causal, 0.3)
    kb, vb = np.broadcast_to(k, q.shape).copy(), np.broadcast_to(v, q.shape).copy()
    ref_out, ref_lse = brute_mha(q, kb, vb, causal, 0.3)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Hq,Hkv", [(8, 4), (4, 2), (6, 3), (16, 1), (16, 4), (3, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_group_map_is_contiguous(Hq, Hkv, causal):
    """SQA(Hq, Hkv) equals MHA on K, V with each KV head repeated g times in place:
    query head h reads KV head floor(h / g) (contiguous groups)."""
    N, dh = 17, 16
    q, k, v = rand((1, N, Hq, dh), 7), rand((1, N, Hkv, dh), 8), rand((1, N, Hkv, dh), 9)
    g = Hq // Hkv
    out, lse = oracle.sqa_fwd(q, k, v, causal, None)
    ref_out, ref_lse = brute_mha(q, np.repeat(k, g, axis=2), np.repeat(v, g, axis=2), causal, dh ** -0.5)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_values(causal):
    """Q = 0 makes every visible score equal, so O_i is the mean of the visible
    V rows and lse_i = ln(#visible keys)."""
    B, N, Hq, Hkv, dh = 2, 29, 4, 2, 16
    q = np.zeros((B, N, Hq, dh))
    k, v = rand((B, N, Hkv, dh), 10), rand((B, N, Hkv, dh), 11)
    out, lse = oracle.sqa_fwd(q, k, v, causal, None)
    g = Hq // Hkv
    for h in range(Hq):
        vh = v[:, :, h // g, :]
        if causal:
            ref = np.cumsum(vh, axis=1) / np.arange(1, N + 1)[None, :, None]
            ref_lse = np.log(np.arange(1, N + 1))
        else:
            ref = np.broadcast_to(vh.mean(axis=1, keepdims=True), vh.shape)
            ref_lse = np.full(N, np.log(N))
        np.testing.assert_allclose(out[:, :, h, :], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, h, :], np.broadcast_to(ref_lse, (B, N)), rtol=0, atol=1e-12)


def test_noncausal_permutation_equivariance():
    B, N, Hq, Hkv, dh = 1, 31, 4, 2, 16
    q, k, v = rand((B, N, Hq, dh), 12), rand((B, N, Hkv, dh), 13), rand((B, N, Hkv, dh), 14)
    perm = np.random.default_rng(15).permutation(N)
    out, lse = oracle.sqa_fwd(q, k, v, False, None)
    out_p, lse_p = oracle.sqa_fwd(q[:, perm], k[:, perm], v[:, perm], False, None)
    np.testing.assert_allclose(out_p, out[:, perm], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_p, lse[:, :, perm], rtol=0, atol=1e-12)
    # Permuting only the keys and values (jointly) leaves the output unchanged.
    out_kv, lse_kv = oracle.sqa_fwd(q, k[:, perm], v[:, perm], False, None)
    np.testing.assert_allclose(out_kv, out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_kv, lse, rtol=0, atol=1e-12)


def test_scale_enters_scores_once():
    """Doubling the scale equals doubling Q (the scale multiplies Q K^T once)."""
    q, k, v = rand((1, 9, 2, 16), 16), rand((1, 9, 1, 16), 17), rand((1, 9, 1, 16), 18)
    a, la = oracle.sqa_fwd(q, k, v, True, 0.5)
    b, lb = oracle.sqa_fwd(2 * q, k, v, True, 0.25)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(la, lb, rtol=0, atol=1e-12)


def _loss(q, k, v, dout, causal, scale):
    out, _ = oracle.sqa_fwd(q, k, v, causal, scale)
    return float(np.sum(out * dout))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,Hq,Hkv", [(5, 4, 2), (17, 4, 2), (6, 3, 1)])
def test_backward_matches_central_differences(causal, N, Hq, Hkv):
    dh, scale, eps = 16, 0.3, 1e-6
    q, k, v = rand((1, N, Hq, dh), 20), rand((1, N, Hkv, dh), 21), rand((1, N, Hkv, dh), 22)
    dout = rand((1, N, Hq, dh), 23)
    dq, dk, dv = oracle.sqa_bwd(q, k, v, dout, causal, scale)
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        flat = x.reshape(-1)
        for t in range(flat.size):
            old = flat[t]
            flat[t] = old + eps
            lp = _loss(q, k, v, dout, causal, scale)
            flat[t] = old - eps
            lm = _loss(q, k, v, dout, causal, scale)
            flat[t] = old
            fd.reshape(-1)[t] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(fd - grad)) / max(1.0, np.max(np.abs(grad)))
        assert err < 1e-7, f"d{name}: finite-difference mismatch {err}"


@pytest.mark.parametrize("causal", [False, True])
def test_backward_conservation_sums(causal):
    """Rows of P sum to 1, so sum_j dV_j = sum over the group of sum_i dO_i;
    rows of dS sum to 0, so sum_j dK_j = 0."""
    B, N, Hq, Hkv, dh = 2, 21, 8, 4, 16
    q, k, v = rand((B, N, Hq, dh), 24), rand((B, N, Hkv, dh), 25), rand((B, N, Hkv, dh), 26)
    dout = rand((B, N, Hq, dh), 27)
    _, dk, dv = oracle.sqa_bwd(q, k, v, dout, causal, None)
    g = Hq // Hkv
    ref_dv = dout.sum(axis=1).reshape(B, Hkv, g, dh).sum(axis=2)
    np.testing.assert_allclose(dv.sum(axis=1), ref_dv, rtol=0, atol=1e-10)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, rtol=0, atol=1e-10)


def test_mha_backward_matches_brute_force_autograd():
    """For H_q = H_kv the backward equals torch autograd of the per-head
    brute-force attention in fp64."""
    import torch

    B, N, H, dh = 1, 13, 2, 16
    q, k, v, dout = (rand((B, N, H, dh), s) for s in (30, 31, 32, 33))
    for causal in (False, True):
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        S = torch.einsum("bihd,bjhd->bhij", tq, tk) * 0.25
        if causal:
            S = S.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
        O = torch.einsum("bhij,bjhd->bihd", torch.softmax(S, dim=-1), tv)
        (O * torch.tensor(dout)).sum().backward()
        dq, dk, dv = oracle.sqa_bwd(q, k, v, dout, causal, 0.25)
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_row_entry_points_agree_with_full(causal):
    B, N, Hq, Hkv, dh = 2, 40, 8, 2, 16
    q, k, v = rand((B, N, Hq, dh), 40), rand((B, N, Hkv, dh), 41), rand((B, N, Hkv, dh), 42)
    dout = rand((B, N, Hq, dh), 43)
    out, lse = oracle.sqa_fwd(q, k, v, causal, None)
    dq, dk, dv = oracle.sqa_bwd(q, k, v, dout, causal, None)
    rng = np.random.default_rng(44)
    qrows = np.stack([rng.integers(0, B, 25), rng.integers(0, N, 25), rng.integers(0, Hq, 25)], 1)
    krows = np.stack([rng.integers(0, B, 25), rng.integers(0, N, 25), rng.integers(0, Hkv, 25)], 1)
    o_r, l_r = oracle.sqa_fwd_rows(q, k, v, qrows, causal, None)
    np.testing.assert_array_equal(o_r, out[qrows[:, 0], qrows[:, 1], qrows[:, 2]])
    np.testing.assert_array_equal(l_r, lse[qrows[:, 0], qrows[:, 2], qrows[:, 1]])
    dq_r, dk_r, dv_r = oracle.sqa_bwd_rows(q, k, v, dout, qrows, krows, causal, None)
    np.testing.assert_allclose(dq_r, dq[qrows[:, 0], qrows[:, 1], qrows[:, 2]], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dk_r, dk[krows[:, 0], krows[:, 1], krows[:, 2]], rtol=0, atol=1e-13)
    np.testing.assert_allclose(dv_r, dv[krows[:, 0], krows[:, 1], krows[:, 2]], rtol=0, atol=1e-13)


def test_invalid_arguments_are_rejected():
    q, k = rand((1, 4, 3, 16), 1), rand((1, 4, 2, 16), 2)
    with pytest.raises(ValueError):
        oracle.sqa_fwd(q, k, k, False, None)  # 3 query heads do not split over 2 KV heads


def test_bf16_inputs_convert_exactly():
    """The generator's bf16 tensors reach the oracle with their exact values."""
    q, k, v, _ = make_inputs(1, 8, 2, 1, 16, seed=3)
    out_bf, lse_bf = oracle.sqa_fwd(q, k, v, True, None)
    out_np, lse_np = oracle.sqa_fwd(q.float().numpy(), k.float().numpy(), v.float().numpy(), True, None)
    np.testing.assert_array_equal(out_bf, out_np)
    np.testing.assert_array_equal(lse_bf, lse_np)


def test_seeded_inputs_are_reproducible():
    a = make_inputs(2, 16, 4, 2, 16, seed=5, with_dout=True)
    b = make_inputs(2, 16, 4, 2, 16, seed=5, with_dout=True)
    import torch

    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and torch.equal(x, y)


def test_head_split_reading_matches_printed_parameter_counts():
    """Rebuild the model card's parameter totals with dh = dim / head_split.
    The reading dh = dim / H_q instead would make SQA's attention larger than
    GQA's, against the card's ordering."""
    with open(os.path.join(GOLDEN, "sqat_m_param_counts.json")) as f:
        g = json.load(f)
    a = g["architecture"]
    d, L, H = a["dim"], a["layers"], a["head_split"]

    def total(hq, hkv, dh):
        attn = d * hq * dh + 2 * d * hkv * dh + hq * dh * d
        layer = attn + 3 * d * a["swiglu_hidden"] + a["norms_per_layer"] * d
        return 2 * a["vocab"] * d + L * layer + d

    for name, (hq, hkv) in g["heads"].items():
        got = total(hq, hkv, d // H) / 1e6
        want = g["printed_params_millions"][name]
        assert abs(got - want) / want < 0.01, (name, got, want)
    counts = {n: total(*hk, d // H) for n, hk in g["heads"].items()}
    assert counts["MHA"] > counts["GQA"] > counts["MQA"] > counts["SQA"]
    assert total(8, 4, d // 8) > counts["GQA"]  # dh = d / H_q contradicts the card
