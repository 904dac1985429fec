"""Pins of the oracle's SQAT-m decoder block (RMSNorm, SQA layer, SwiGLU
feed-forward, pre-norm residuals), CPU only.

Each test fixes the result by something other than the oracle itself: closed
forms (unit RMS after normalisation, the SwiGLU product for scalars, a block
with zero output projections is the identity), invariances (scaling the
input of RMSNorm without eps), the card's printed parameter totals, an
independent torch implementation differentiated by autograd, and central
finite differences.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle.block import EPS, block_bwd, block_fwd, rmsnorm, rmsnorm_bwd, silu, swiglu_bwd, swiglu_fwd

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _params(rng, d, Hq, Hkv, dh, hidden, s=0.2):
    return {"g1": 1.0 + 0.1 * rng.standard_normal(d), "g2": 1.0 + 0.1 * rng.standard_normal(d),
            "wq": rng.standard_normal((d, Hq * dh)) * s, "wk": rng.standard_normal((d, Hkv * dh)) * s,
            "wv": rng.standard_normal((d, Hkv * dh)) * s, "wo": rng.standard_normal((Hq * dh, d)) * s,
            "w1": rng.standard_normal((d, hidden)) * s, "w3": rng.standard_normal((d, hidden)) * s,
            "w2": rng.standard_normal((hidden, d)) * s}


def test_rmsnorm_gives_unit_rms_and_ignores_input_scale():
    x = np.random.default_rng(0).standard_normal((3, 7, 32)) * 5
    y = rmsnorm(x, np.ones(32), eps=0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(rmsnorm(3.7 * x, np.ones(32), eps=0.0), y, rtol=1e-13)
    g = np.arange(1, 33, dtype=np.float64)
    np.testing.assert_allclose(rmsnorm(x, g, eps=0.0), y * g, rtol=1e-14)
    # eps matters only next to tiny inputs
    small = np.full((1, 4), 1e-4)
    assert rmsnorm(small, np.ones(4))[0, 0] == pytest.approx(1e-4 / math.sqrt(1e-8 + EPS), rel=1e-12)


def test_swiglu_of_scalars_and_of_zero():
    w1, w3, w2 = np.array([[2.0]]), np.array([[-3.0]]), np.array([[0.5]])
    for u in (-1.3, 0.0, 0.7):
        a = 2.0 * u
        assert swiglu_fwd(np.array([[u]]), w1, w3, w2)[0, 0] == pytest.approx(
            0.5 * (a / (1 + math.exp(-a))) * (-3.0 * u), abs=1e-15)
    assert silu(np.array(0.0)) == 0.0
    rng = np.random.default_rng(1)
    z = swiglu_fwd(np.zeros((2, 8)), rng.standard_normal((8, 12)), rng.standard_normal((8, 12)),
                   rng.standard_normal((12, 8)))
    assert np.all(z == 0)


def test_block_with_zero_output_projections_is_the_identity():
    rng = np.random.default_rng(2)
    p = _params(rng, 16, 4, 2, 4, 24)
    p["wo"][:] = 0
    p["w2"][:] = 0
    x = rng.standard_normal((2, 9, 16))
    np.testing.assert_array_equal(block_fwd(x, p, 4, 2), x)


def test_block_weights_match_the_printed_parameter_totals():
    with open(os.path.join(GOLDEN, "sqat_m_param_counts.json")) as f:
        g = json.load(f)
    a = g["architecture"]
    d, dh = a["dim"], a["dim"] // a["head_split"]
    for name, (hq, hkv) in g["heads"].items():
        p = _params(np.random.default_rng(0), d, hq, hkv, dh, a["swiglu_hidden"])
        per_layer = sum(v.size for v in p.values())
        total = a["layers"] * per_layer + 2 * a["vocab"] * d + d  # embeddings, head, final norm
        want = g["printed_params_millions"][name]
        assert abs(total / 1e6 - want) / want < 0.01, (name, total)


def _torch_block(x, p, Hq, Hkv, causal, base):
    def rms(t, gg):
        return t * torch.rsqrt((t * t).mean(-1, keepdim=True) + EPS) * gg

    B, N, d = x.shape
    dh = p["wq"].shape[1] // Hq
    u = rms(x, p["g1"])
    q = (u @ p["wq"]).reshape(B, N, Hq, dh)
    k = (u @ p["wk"]).reshape(B, N, Hkv, dh)
    v = (u @ p["wv"]).reshape(B, N, Hkv, dh)
    theta = base ** (-torch.arange(0, dh, 2, dtype=torch.float64) / dh)
    rot = torch.polar(torch.ones(N, dh // 2, dtype=torch.float64),
                      torch.arange(N, dtype=torch.float64)[:, None] * theta[None, :])[None, :, None, :]

    def turn(t):
        return torch.view_as_real(torch.view_as_complex(t.reshape(*t.shape[:-1], dh // 2, 2).contiguous()) * rot
                                  ).reshape(t.shape)

    q, k = turn(q), turn(k)
    g = Hq // Hkv
    k, v = k.repeat_interleave(g, dim=2), v.repeat_interleave(g, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(dh)
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, -1), v).reshape(B, N, Hq * dh)
    h = x + o @ p["wo"]
    w = rms(h, p["g2"])
    return h + (torch.nn.functional.silu(w @ p["w1"]) * (w @ p["w3"])) @ p["w2"]


@pytest.mark.parametrize("Hq,Hkv,dh,causal", [(8, 4, 4, True), (4, 1, 8, False), (4, 4, 8, True)])
def test_block_matches_independent_autograd(Hq, Hkv, dh, causal):
    rng = np.random.default_rng(Hq + dh)
    B, N, d, hidden = 2, 11, 16, 24
    p = _params(rng, d, Hq, Hkv, dh, hidden)
    x = rng.standard_normal((B, N, d))
    dy = rng.standard_normal((B, N, d))
    y = block_fwd(x, p, Hq, Hkv, causal)
    dx, grads = block_bwd(x, p, dy, Hq, Hkv, causal)
    tx = torch.tensor(x, requires_grad=True)
    tp = {k: torch.tensor(v, requires_grad=True) for k, v in p.items()}
    ty = _torch_block(tx, tp, Hq, Hkv, causal, 10000.0)
    (ty * torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(y, ty.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dx, tx.grad.numpy(), rtol=0, atol=1e-11)
    for k in p:
        np.testing.assert_allclose(grads[k], tp[k].grad.numpy(), rtol=0, atol=1e-11, err_msg=k)


def test_norm_and_ffn_gradients_match_central_differences():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 10))
    g = 1 + 0.2 * rng.standard_normal(10)
    dy = rng.standard_normal((3, 10))
    dx, dg = rmsnorm_bwd(x, g, dy)
    w1, w3, w2 = rng.standard_normal((10, 6)), rng.standard_normal((10, 6)), rng.standard_normal((6, 10))
    du, dw1, dw3, dw2 = swiglu_bwd(x, w1, w3, w2, dy)
    eps = 1e-6
    checks = [
        (lambda t: float((rmsnorm(t, g) * dy).sum()), x, dx),
        (lambda t: float((rmsnorm(x, t) * dy).sum()), g, dg),
        (lambda t: float((swiglu_fwd(t, w1, w3, w2) * dy).sum()), x, du),
        (lambda t: float((swiglu_fwd(x, t, w3, w2) * dy).sum()), w1, dw1),
        (lambda t: float((swiglu_fwd(x, w1, t, w2) * dy).sum()), w3, dw3),
        (lambda t: float((swiglu_fwd(x, w1, w3, t) * dy).sum()), w2, dw2),
    ]
    for f, t, grad in checks:
        u = rng.standard_normal(t.shape)
        fd = (f(t + eps * u) - f(t - eps * u)) / (2 * eps)
        assert fd == pytest.approx(float((grad * u).sum()), rel=1e-6, abs=1e-8)
