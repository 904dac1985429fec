"""Pins of the oracle's full SQA layer (reduced-width projections, rotary
embedding, attention core), CPU only.

Each test fixes the result by something other than the oracle itself: closed
forms of the rotation, its invariances (orthogonal, relative-position), the
reduction of the layer to the bare core, the card's printed parameter totals
(which fix the projection widths), an independent torch implementation
differentiated by autograd (rotation by complex multiplication, softmax
attention by brute force), and central finite differences.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.layer import rope, rope_angles, sqa_layer_bwd, sqa_layer_fwd

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _weights(rng, d, Hq, Hkv, dh, s=0.2):
    return (rng.standard_normal((d, Hq * dh)) * s, rng.standard_normal((d, Hkv * dh)) * s,
            rng.standard_normal((d, Hkv * dh)) * s, rng.standard_normal((Hq * dh, d)) * s)


# ----------------------------------------------------------------------------- rotation


def test_rotation_at_position_zero_is_the_identity():
    x = np.random.default_rng(0).standard_normal((2, 1, 3, 16))
    np.testing.assert_array_equal(rope(x), x)


def test_two_channel_head_turns_by_the_position_in_radians():
    # dh = 2: one pair with theta_0 = base^0 = 1, so token m turns by m radians
    x = np.zeros((1, 5, 1, 2))
    x[..., 0] = 1.0
    y = rope(x)
    for m in range(5):
        np.testing.assert_allclose(y[0, m, 0], [math.cos(m), math.sin(m)], atol=1e-15)


def test_pair_j_turns_with_frequency_base_to_minus_2j_over_dh():
    dh, base = 8, 10000.0
    for j in range(dh // 2):
        x = np.zeros((1, 2, 1, dh))
        x[..., 2 * j] = 1.0  # unit vector in the first channel of pair j
        y = rope(x)[0, 1, 0]
        ang = math.atan2(y[2 * j + 1], y[2 * j])
        assert ang == pytest.approx(base ** (-2 * j / dh), abs=1e-14)
        others = np.delete(y, [2 * j, 2 * j + 1])
        assert np.all(others == 0)


def test_rotation_is_orthogonal_and_inverted_by_the_opposite_angle():
    x = np.random.default_rng(1).standard_normal((2, 50, 3, 16))
    y = rope(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(rope(y, inverse=True), x, atol=1e-13)


def test_scores_depend_only_on_the_relative_position():
    rng = np.random.default_rng(2)
    dh = 16
    qv, kv = rng.standard_normal(dh), rng.standard_normal(dh)

    def score(m, n):
        q = np.zeros((1, max(m, n) + 1, 1, dh))
        k = np.zeros_like(q)
        q[0, m, 0], k[0, n, 0] = qv, kv
        return float(rope(q)[0, m, 0] @ rope(k)[0, n, 0])

    for m, n, shift in [(7, 3, 11), (3, 7, 5), (20, 20, 9)]:
        assert score(m + shift, n + shift) == pytest.approx(score(m, n), abs=1e-12)
    assert score(5, 5) == pytest.approx(float(qv @ kv), abs=1e-12)
    assert rope_angles(3, 4).shape == (3, 2)


# ----------------------------------------------------------------------------- layer


def test_layer_with_identity_weights_and_no_rotation_is_the_core():
    rng = np.random.default_rng(3)
    B, N, H, dh = 2, 20, 4, 8
    d = H * dh
    x = rng.standard_normal((B, N, d))
    eye = np.eye(d)
    y, _ = sqa_layer_fwd(x, eye, eye, eye, eye, H, H, causal=True, rope_base=None)
    qkv = x.reshape(B, N, H, dh)
    out, _ = oracle.sqa_fwd(qkv, qkv, qkv, True)
    np.testing.assert_allclose(y, out.reshape(B, N, d), atol=1e-13)


def test_printed_totals_fix_the_projection_widths():
    """The card prints totals rounded to 0.1M.  Their differences between head
    layouts come only from the attention weights (the rest of the model is the
    same), so they fix d*H_q*dh + 2*d*H_kv*dh + H_q*dh*d per layer: the query
    and output projections shrink with H_q, the key and value ones with H_kv."""
    with open(os.path.join(GOLDEN, "sqat_m_param_counts.json")) as f:
        g = json.load(f)
    a = g["architecture"]
    d, L, dh = a["dim"], a["layers"], a["dim"] // a["head_split"]
    rng = np.random.default_rng(0)

    def attn_params(hq, hkv):
        return sum(w.size for w in _weights(rng, d, hq, hkv, dh))

    printed = g["printed_params_millions"]
    for name, (hq, hkv) in g["heads"].items():
        diff = L * (attn_params(16, 16) - attn_params(hq, hkv)) / 1e6
        assert abs(diff - (printed["MHA"] - printed[name])) <= 0.1 + 1e-9, (name, diff)
    # the other reading (W_o of full width d -> d) would change the SQA total by 8*d*d*(1 - 1/2)
    full_wo = L * (attn_params(16, 16) - attn_params(8, 4) - d * d // 2) / 1e6
    assert abs(full_wo - (printed["MHA"] - printed["SQA"])) > 0.2


def _torch_layer(x, wq, wk, wv, wo, Hq, Hkv, causal, base):
    """Independent reference: complex-number rotation, brute-force softmax attention."""
    B, N, d = x.shape
    dh = wq.shape[1] // Hq
    q = (x @ wq).reshape(B, N, Hq, dh)
    k = (x @ wk).reshape(B, N, Hkv, dh)
    v = (x @ wv).reshape(B, N, Hkv, dh)
    if base is not None:
        theta = base ** (-torch.arange(0, dh, 2, dtype=torch.float64) / dh)
        rot = torch.polar(torch.ones(N, dh // 2, dtype=torch.float64),
                          torch.arange(N, dtype=torch.float64)[:, None] * theta[None, :])[None, :, None, :]

        def turn(t):
            c = torch.view_as_complex(t.reshape(*t.shape[:-1], dh // 2, 2).contiguous()) * rot
            return torch.view_as_real(c).reshape(t.shape)

        q, k = turn(q), turn(k)
    g = Hq // Hkv
    k = k.repeat_interleave(g, dim=2)
    v = v.repeat_interleave(g, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(dh)
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, dim=-1), v)
    return o.reshape(B, N, Hq * dh) @ wo


@pytest.mark.parametrize("Hq,Hkv,dh,causal,base", [(8, 4, 16, True, 10000.0), (4, 1, 8, False, 10000.0),
                                                   (4, 4, 16, True, None), (6, 2, 32, True, 500.0)])
def test_layer_matches_independent_autograd(Hq, Hkv, dh, causal, base):
    rng = np.random.default_rng(Hq * 10 + dh)
    B, N, d = 2, 17, 24
    x = rng.standard_normal((B, N, d))
    ws = _weights(rng, d, Hq, Hkv, dh)
    dy = rng.standard_normal((B, N, d))
    y, _ = sqa_layer_fwd(x, *ws, Hq, Hkv, causal=causal, rope_base=base)
    grads = sqa_layer_bwd(x, *ws, dy, Hq, Hkv, causal=causal, rope_base=base)

    tx = torch.tensor(x, requires_grad=True)
    tws = [torch.tensor(w, requires_grad=True) for w in ws]
    ty = _torch_layer(tx, *tws, Hq, Hkv, causal, base)
    (ty * torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(y, ty.detach().numpy(), rtol=0, atol=1e-12)
    for got, ref in zip(grads, [tx.grad] + [w.grad for w in tws]):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-11)


def test_layer_gradients_match_central_differences():
    rng = np.random.default_rng(9)
    B, N, d, Hq, Hkv, dh = 1, 9, 12, 4, 2, 8
    x = rng.standard_normal((B, N, d))
    ws = list(_weights(rng, d, Hq, Hkv, dh, s=0.3))
    dy = rng.standard_normal((B, N, d))
    grads = sqa_layer_bwd(x, *ws, dy, Hq, Hkv, causal=True)
    params = [x] + ws

    def loss(ps):
        return float((sqa_layer_fwd(ps[0], *ps[1:], Hq, Hkv, causal=True)[0] * dy).sum())

    eps = 1e-6
    for i, gr in enumerate(grads):
        u = rng.standard_normal(params[i].shape)
        plus = [p.copy() for p in params]
        minus = [p.copy() for p in params]
        plus[i] = plus[i] + eps * u
        minus[i] = minus[i] - eps * u
        fd = (loss(plus) - loss(minus)) / (2 * eps)
        assert fd == pytest.approx(float((gr * u).sum()), rel=1e-6, abs=1e-7), i


def test_layer_rejects_mismatched_weights():
    x = np.zeros((1, 4, 8))
    with pytest.raises(ValueError):
        sqa_layer_fwd(x, np.zeros((8, 16)), np.zeros((8, 8)), np.zeros((8, 8)), np.zeros((8, 8)), 4, 2)
    with pytest.raises(ValueError):
        sqa_layer_fwd(x, np.zeros((8, 16)), np.zeros((8, 8)), np.zeros((8, 8)), np.zeros((16, 8)), 4, 3)
