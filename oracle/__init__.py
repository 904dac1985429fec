"""fp64 CPU oracle for Sparse Query Attention -- TEST INFRASTRUCTURE ONLY.

This package is the yardstick the CUDA library is checked against.  Only the
test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it.  It shares no code with the CUDA path, and the
library never calls it.

The attention arithmetic lives in ``sqa_oracle.c`` (plain loops in fp64,
OpenMP over rows).  This module only builds that file with gcc and marshals
numpy arrays.  Inputs are converted to fp64 before the call; bf16 values
convert exactly.  ``layer.py`` adds the full layer around that core
(projections and rotary embedding, in numpy fp64), ``block.py`` one decoder
block around the layer (RMSNorm, SwiGLU feed-forward, residuals).

What is computed follows the SQAT-m model card ("Architecture details": 16
heads for the dimension split, 8 query groups, 4 key/value groups; "Model size
difference": reduced query and output projections), the arXiv 2510.01817
abstract (query heads are reduced, score FLOPs fall with them) and the GQA
summary ("The idea": query heads split into groups that share one key head and
one value head; GQA-1 is MQA, GQA-H is MHA).  See ``sqa_oracle.c`` for the
formulas.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sqa_oracle.c")
_LIB = os.path.join(_HERE, "libsqa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile sqa_oracle.c into libsqa_oracle.so with gcc (-O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        base = [dp, dp, dp, i64, i64, i64, i64, i64, ctypes.c_int, ctypes.c_double]
        lib.sqa_oracle_fwd.argtypes = base + [dp, dp]
        lib.sqa_oracle_fwd_rows.argtypes = base + [ip, i64, dp, dp]
        bbase = [dp, dp, dp, dp, i64, i64, i64, i64, i64, ctypes.c_int, ctypes.c_double]
        lib.sqa_oracle_bwd.argtypes = bbase + [dp, dp, dp]
        lib.sqa_oracle_bwd_rows.argtypes = bbase + [ip, i64, dp, ip, i64, dp, dp]
        lib.sqa_oracle_decode.argtypes = [dp, dp, dp, ip, i64, i64, i64, i64, i64, ctypes.c_double, dp, dp]
        for f in (lib.sqa_oracle_fwd, lib.sqa_oracle_fwd_rows, lib.sqa_oracle_bwd, lib.sqa_oracle_bwd_rows,
                  lib.sqa_oracle_decode):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):  # a torch tensor (any dtype, CPU or GPU)
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray, t=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(t))


def _shape(q, k):
    B, N, Hq, dh = q.shape
    Bk, Nk, Hkv, dhk = k.shape
    if (Bk, Nk, dhk) != (B, N, dh):
        raise ValueError("q and k/v shapes disagree")
    return B, N, Hq, Hkv, dh


def _scale(scale, dh):
    return float(scale) if scale is not None and scale > 0 else 1.0 / np.sqrt(dh)


def _check(rc):
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (code {rc})")


def sqa_fwd(q, k, v, causal: bool, scale: float | None = None):
    """Full forward.  q [B,N,Hq,dh], k/v [B,N,Hkv,dh] -> (out [B,N,Hq,dh], lse [B,Hq,N]), fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N, Hq, Hkv, dh = _shape(q, k)
    out = np.zeros((B, N, Hq, dh))
    lse = np.zeros((B, Hq, N))
    _check(_load().sqa_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), B, N, Hq, Hkv, dh, int(causal),
                                  _scale(scale, dh), _ptr(out), _ptr(lse)))
    return out, lse


def sqa_fwd_rows(q, k, v, rows, causal: bool, scale: float | None = None):
    """Forward for selected query rows.  rows: int array [n,3] of (b, i, h).
    Returns (out_rows [n,dh], lse_rows [n])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N, Hq, Hkv, dh = _shape(q, k)
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    out = np.zeros((rows.shape[0], dh))
    lse = np.zeros(rows.shape[0])
    _check(_load().sqa_oracle_fwd_rows(_ptr(q), _ptr(k), _ptr(v), B, N, Hq, Hkv, dh, int(causal),
                                       _scale(scale, dh), _ptr(rows, ctypes.c_int64), rows.shape[0],
                                       _ptr(out), _ptr(lse)))
    return out, lse


def sqa_bwd(q, k, v, dout, causal: bool, scale: float | None = None):
    """Full backward of L = sum(dout * O).  Returns (dq, dk, dv) in fp64."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, Hq, Hkv, dh = _shape(q, k)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    _check(_load().sqa_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, N, Hq, Hkv, dh, int(causal),
                                  _scale(scale, dh), _ptr(dq), _ptr(dk), _ptr(dv)))
    return dq, dk, dv


def sqa_bwd_rows(q, k, v, dout, qrows, krows, causal: bool, scale: float | None = None):
    """Backward for selected rows: dQ for qrows (b, i, h) and dK, dV for krows (b, j, kvh)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, N, Hq, Hkv, dh = _shape(q, k)
    qrows = np.ascontiguousarray(qrows, dtype=np.int64).reshape(-1, 3)
    krows = np.ascontiguousarray(krows, dtype=np.int64).reshape(-1, 3)
    dq = np.zeros((qrows.shape[0], dh))
    dk = np.zeros((krows.shape[0], dh))
    dv = np.zeros((krows.shape[0], dh))
    _check(_load().sqa_oracle_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, N, Hq, Hkv, dh,
                                       int(causal), _scale(scale, dh), _ptr(qrows, ctypes.c_int64),
                                       qrows.shape[0], _ptr(dq), _ptr(krows, ctypes.c_int64),
                                       krows.shape[0], _ptr(dk), _ptr(dv)))
    return dq, dk, dv


def sqa_decode(q, k, v, lens=None, scale: float | None = None):
    """Decoding step: q [B,Hq,dh] (one token per sequence) against the first
    lens[b] entries of the cache k/v [B,N,Hkv,dh] (all N when lens is None).
    Returns (out [B,Hq,dh], lse [B,Hq]) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, dh = q.shape
    Bk, N, Hkv, dhk = k.shape
    if (Bk, dhk) != (B, dh) or v.shape != k.shape:
        raise ValueError("q and k/v shapes disagree")
    lens = np.full(B, N, dtype=np.int64) if lens is None else np.ascontiguousarray(lens, dtype=np.int64)
    out = np.zeros((B, Hq, dh))
    lse = np.zeros((B, Hq))
    _check(_load().sqa_oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(lens, ctypes.c_int64), B, N, Hq, Hkv, dh,
                                     _scale(scale, dh), _ptr(out), _ptr(lse)))
    return out, lse
