"""fp64 CPU oracle of one SQAT-m decoder block -- TEST INFRASTRUCTURE ONLY.

Like the rest of ``oracle/``, this is a yardstick for tests and is never
called by the library.  The SQAT-m model card ("Architecture details") lists
the parts of a layer: Sparse Query Attention, a SwiGLU feed-forward of hidden
width 768, RoPE and RMS normalisation.  It gives no order, so the plain
pre-norm residual reading is taken:

    h = x + SQA(RMSNorm(x; g1))
    y = h + FFN(RMSNorm(h; g2)),   FFN(u) = (silu(u W1) * (u W3)) W2

with RMSNorm(x; g) = g * x / sqrt(mean(x^2) + eps) over the model dimension,
eps = 1e-6, silu(a) = a / (1 + exp(-a)), W1, W3 [d, hidden], W2 [hidden, d],
no biases (two norms and 3 d hidden FFN weights per layer meet the card's
parameter totals).  SQA is ``oracle.layer.sqa_layer_fwd``.  The backward of
L = sum(dY * Y) is written out step by step; matrix products are numpy's.
"""
from __future__ import annotations

import numpy as np

from .layer import ROPE_BASE, sqa_layer_bwd, sqa_layer_fwd

EPS = 1e-6


def rmsnorm(x, g, eps: float = EPS) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * np.asarray(g, dtype=np.float64)


def rmsnorm_bwd(x, g, dy, eps: float = EPS):
    """Gradients (dx, dg) of sum(dy * rmsnorm(x, g))."""
    x, g, dy = (np.asarray(a, dtype=np.float64) for a in (x, g, dy))
    d = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xhat = x * r
    dg = (dy * xhat).reshape(-1, d).sum(axis=0)
    dxhat = dy * g
    # xhat = x r with dr/dx = -r^3 x / d
    dx = r * dxhat - (r ** 3) * x * np.sum(dxhat * x, axis=-1, keepdims=True) / d
    return dx, dg


def silu(a):
    return a / (1.0 + np.exp(-a))


def swiglu_fwd(u, w1, w3, w2) -> np.ndarray:
    u = np.asarray(u, dtype=np.float64)
    return (silu(u @ w1) * (u @ w3)) @ w2


def swiglu_bwd(u, w1, w3, w2, dy):
    """Gradients (du, dW1, dW3, dW2) of sum(dy * swiglu_fwd(u, ...))."""
    u, w1, w3, w2, dy = (np.asarray(a, dtype=np.float64) for a in (u, w1, w3, w2, dy))
    d = u.shape[-1]
    uf, dyf = u.reshape(-1, d), dy.reshape(-1, w2.shape[1])
    a, b = uf @ w1, uf @ w3
    s = 1.0 / (1.0 + np.exp(-a))
    act = a * s
    m = act * b
    dw2 = m.T @ dyf
    dm = dyf @ w2.T
    db = dm * act
    da = dm * b * (s + a * s * (1.0 - s))  # silu'(a) = s + a s (1 - s)
    dw1, dw3 = uf.T @ da, uf.T @ db
    du = (da @ w1.T + db @ w3.T).reshape(u.shape)
    return du, dw1, dw3, dw2


def block_fwd(x, p: dict, Hq: int, Hkv: int, causal: bool = True, rope_base: float | None = ROPE_BASE):
    """y [B, N, d] of one block.  p: g1, g2 [d]; wq, wk, wv, wo (see
    ``oracle.layer``); w1, w3 [d, hidden]; w2 [hidden, d]."""
    x = np.asarray(x, dtype=np.float64)
    a, _ = sqa_layer_fwd(rmsnorm(x, p["g1"]), p["wq"], p["wk"], p["wv"], p["wo"], Hq, Hkv, causal,
                         rope_base=rope_base)
    h = x + a
    return h + swiglu_fwd(rmsnorm(h, p["g2"]), p["w1"], p["w3"], p["w2"])


def block_bwd(x, p: dict, dy, Hq: int, Hkv: int, causal: bool = True, rope_base: float | None = ROPE_BASE):
    """Gradients of sum(dY * block_fwd(x, p)): (dx, dict of parameter gradients)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    n1 = rmsnorm(x, p["g1"])
    a, _ = sqa_layer_fwd(n1, p["wq"], p["wk"], p["wv"], p["wo"], Hq, Hkv, causal, rope_base=rope_base)
    h = x + a
    n2 = rmsnorm(h, p["g2"])
    # y = h + FFN(n2)
    dn2, dw1, dw3, dw2 = swiglu_bwd(n2, p["w1"], p["w3"], p["w2"], dy)
    dh_norm, dg2 = rmsnorm_bwd(h, p["g2"], dn2)
    dh = dy + dh_norm
    # h = x + SQA(n1)
    dn1, dwq, dwk, dwv, dwo = sqa_layer_bwd(n1, p["wq"], p["wk"], p["wv"], p["wo"], dh, Hq, Hkv, causal,
                                           rope_base=rope_base)
    dx_norm, dg1 = rmsnorm_bwd(x, p["g1"], dn1)
    grads = {"g1": dg1, "g2": dg2, "wq": dwq, "wk": dwk, "wv": dwv, "wo": dwo, "w1": dw1, "w3": dw3, "w2": dw2}
    return dh + dx_norm, grads
