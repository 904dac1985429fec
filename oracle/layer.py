"""fp64 CPU oracle of the full SQA attention layer -- TEST INFRASTRUCTURE ONLY.

Like the rest of ``oracle/``, this module is the yardstick for tests and is
never called by the library.  It wraps the attention core of
``sqa_oracle.c`` (through ``oracle.sqa_fwd`` / ``oracle.sqa_bwd``) with the
steps on either side of it:

* reduced-width projections (SQAT-m model card, "Model size difference": the
  query projection and the output projection shrink with the query-head count):
  Q = X W_q with W_q [d, H_q*dh], K = X W_k and V = X W_v with W_k, W_v
  [d, H_kv*dh], Y = O W_o with W_o [H_q*dh, d]; no biases (the card's
  parameter totals are met without them); column h*dh + c of W_q is channel c
  of query head h (heads contiguous), likewise for W_k, W_v and the rows of W_o;
* rotary position embedding on Q and K (the card lists "RoPE" and nothing
  more).  The pages fix no variant, so the original rotary form is taken:
  channels (2j, 2j+1) of every head of the token at position i (0-based) are
  turned by the angle i * theta_j, theta_j = base^(-2j/dh), base 10000.

Backward of L = sum(dY * Y): dO = dY W_o^T, dW_o = O^T dY, the core backward
gives the gradients of the rotated Q and K and of V, the rotation is undone
(its transpose turns by -i * theta_j), then dW_q = X^T dQ, dW_k = X^T dK,
dW_v = X^T dV and dX = dQ W_q^T + dK W_k^T + dV W_v^T.  Matrix products are
numpy's (a library primitive as one step); nothing is fused or reordered.
"""
from __future__ import annotations

import numpy as np

from . import sqa_bwd, sqa_fwd

ROPE_BASE = 10000.0


def rope_angles(n_tokens: int, dh: int, base: float = ROPE_BASE, positions=None) -> np.ndarray:
    """Angle [N, dh/2] by which channel pair j of the token at each position turns."""
    if dh % 2:
        raise ValueError("rotary embedding needs an even head dim")
    pos = np.arange(n_tokens, dtype=np.float64) if positions is None else np.asarray(positions, np.float64)
    theta = base ** (-2.0 * np.arange(dh // 2, dtype=np.float64) / dh)
    return pos[:, None] * theta[None, :]


def rope(x, base: float = ROPE_BASE, positions=None, inverse: bool = False) -> np.ndarray:
    """Rotate x [B, N, H, dh]: pair (x[..., 2j], x[..., 2j+1]) of token i by +/- i * theta_j."""
    x = np.asarray(x, dtype=np.float64)
    ang = rope_angles(x.shape[1], x.shape[3], base, positions)
    if inverse:
        ang = -ang
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = a * c - b * s
    y[..., 1::2] = a * s + b * c
    return y


def _project(x, w, heads: int, dh: int) -> np.ndarray:
    B, N, d = x.shape
    if w.shape != (d, heads * dh):
        raise ValueError(f"projection weight must be [{d}, {heads * dh}], got {list(w.shape)}")
    return (x.reshape(B * N, d) @ w).reshape(B, N, heads, dh)


def sqa_layer_fwd(x, wq, wk, wv, wo, Hq: int, Hkv: int, causal: bool = True, scale: float | None = None,
                  rope_base: float | None = ROPE_BASE):
    """Y [B, N, d] of the SQA layer and its intermediates (dict: q, k, v after
    the rotation, out and lse of the core).  rope_base=None leaves Q and K
    unrotated."""
    x = np.asarray(x, dtype=np.float64)
    wq, wk, wv, wo = (np.asarray(w, dtype=np.float64) for w in (wq, wk, wv, wo))
    B, N, d = x.shape
    if Hq % Hkv:
        raise ValueError("H_q must be a multiple of H_kv")
    dh = wq.shape[1] // Hq
    q = _project(x, wq, Hq, dh)
    k = _project(x, wk, Hkv, dh)
    v = _project(x, wv, Hkv, dh)
    if rope_base is not None:
        q, k = rope(q, rope_base), rope(k, rope_base)
    out, lse = sqa_fwd(q, k, v, causal, scale)
    if wo.shape != (Hq * dh, d):
        raise ValueError(f"output weight must be [{Hq * dh}, {d}], got {list(wo.shape)}")
    y = (out.reshape(B * N, Hq * dh) @ wo).reshape(B, N, d)
    return y, {"q": q, "k": k, "v": v, "out": out, "lse": lse}


def sqa_layer_bwd(x, wq, wk, wv, wo, dy, Hq: int, Hkv: int, causal: bool = True, scale: float | None = None,
                  rope_base: float | None = ROPE_BASE):
    """Gradients (dX, dW_q, dW_k, dW_v, dW_o) of L = sum(dY * Y)."""
    x = np.asarray(x, dtype=np.float64)
    wq, wk, wv, wo = (np.asarray(w, dtype=np.float64) for w in (wq, wk, wv, wo))
    dy = np.asarray(dy, dtype=np.float64)
    B, N, d = x.shape
    dh = wq.shape[1] // Hq
    _, mid = sqa_layer_fwd(x, wq, wk, wv, wo, Hq, Hkv, causal, scale, rope_base)
    dyf = dy.reshape(B * N, d)
    dwo = mid["out"].reshape(B * N, Hq * dh).T @ dyf
    dout = (dyf @ wo.T).reshape(B, N, Hq, dh)
    dq, dk, dv = sqa_bwd(mid["q"], mid["k"], mid["v"], dout, causal, scale)
    if rope_base is not None:
        dq, dk = rope(dq, rope_base, inverse=True), rope(dk, rope_base, inverse=True)
    xf = x.reshape(B * N, d)
    dqf, dkf, dvf = dq.reshape(B * N, Hq * dh), dk.reshape(B * N, Hkv * dh), dv.reshape(B * N, Hkv * dh)
    dwq, dwk, dwv = xf.T @ dqf, xf.T @ dkf, xf.T @ dvf
    dx = (dqf @ wq.T + dkf @ wk.T + dvf @ wv.T).reshape(B, N, d)
    return dx, dwq, dwk, dwv, dwo
