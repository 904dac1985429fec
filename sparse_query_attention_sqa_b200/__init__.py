"""Sparse Query Attention on B200 (sm_100a): Python binding of libsqa.so.

Every step of the attention forward and backward runs in the CUDA kernels of
``libsqa.so`` (C ABI in ``include/sqa.h``).  This module only checks tensor
metadata, allocates outputs with PyTorch and passes raw pointers and the
current stream through ctypes.  There is no CPU fallback: if the library is
missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "SqaError", "load_library", "library_path", "sqa_fwd", "sqa_bwd", "bwd_workspace_bytes", "sqa_decode",
    "decode_workspace_bytes",
    "device_status", "timeout_info", "set_timing_events", "Shape", "LayerShape", "layer_workspace_bytes",
    "sqa_layer_fwd", "sqa_layer_bwd", "BlockShape", "block_state_bytes", "sqa_block_fwd", "sqa_block_bwd",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsqa.so")
_lib = None

SQA_OK, SQA_ERR_INVALID_ARG, SQA_ERR_UNSUPPORTED, SQA_ERR_CUDA = 0, 1, 2, 3


class SqaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"[status {status}] {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("H_q", ctypes.c_int), ("H_kv", ctypes.c_int),
                ("dh", ctypes.c_int)]


class LayerShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int), ("H_q", ctypes.c_int),
                ("H_kv", ctypes.c_int), ("dh", ctypes.c_int)]


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libsqa.so (built in-tree by ``build.py``); raises if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libsqa.so is not built ({_LIB_PATH}); run sparse_query_attention_sqa_b200/build.py")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, fp, c_int, c_float, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.sqa_fwd.argtypes = [vp, vp, vp, vp, fp, Shape, c_int, c_float, vp]
    lib.sqa_fwd.restype = c_int
    lib.sqa_fwd_workspace_bytes.argtypes = [Shape, c_int]
    lib.sqa_fwd_workspace_bytes.restype = sz
    lib.sqa_fwd_with_workspace.argtypes = [vp, vp, vp, vp, fp, vp, sz, Shape, c_int, c_float, vp]
    lib.sqa_fwd_with_workspace.restype = c_int
    lib.sqa_bwd_workspace_bytes.argtypes = [Shape]
    lib.sqa_bwd_workspace_bytes.restype = sz
    lib.sqa_bwd.argtypes = [vp, vp, vp, vp, vp, fp, vp, vp, vp, vp, sz, Shape, c_int, c_float, vp]
    lib.sqa_bwd.restype = c_int
    lib.sqa_decode_workspace_bytes.argtypes = [Shape]
    lib.sqa_decode_workspace_bytes.restype = sz
    lib.sqa_decode.argtypes = [vp, vp, vp, vp, vp, fp, vp, sz, Shape, c_float, vp]
    lib.sqa_decode.restype = c_int
    lib.sqa_status_string.argtypes = [c_int]
    lib.sqa_status_string.restype = ctypes.c_char_p
    lib.sqa_last_error.argtypes = []
    lib.sqa_last_error.restype = ctypes.c_char_p
    lib.sqa_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint), c_int]
    lib.sqa_device_status.restype = c_int
    lib.sqa_device_timeout_info.argtypes = [ctypes.POINTER(ctypes.c_uint), c_int]
    lib.sqa_device_timeout_info.restype = c_int
    lib.sqa_set_timing_events.argtypes = [c_int, vp, vp]
    lib.sqa_set_timing_events.restype = c_int
    lib.sqa_layer_workspace_bytes.argtypes = [LayerShape, c_int]
    lib.sqa_layer_workspace_bytes.restype = sz
    lib.sqa_layer_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, fp, vp, sz, LayerShape, c_int, c_float, c_float, vp]
    lib.sqa_layer_fwd.restype = c_int
    lib.sqa_layer_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, fp, vp, fp, fp, vp, sz, LayerShape, c_int, c_float,
                                  c_float, vp]
    lib.sqa_layer_bwd.restype = c_int
    lib.sqa_version.argtypes = []
    lib.sqa_version.restype = c_int
    _lib = lib
    return lib


def _check(status: int):
    if status != SQA_OK:
        lib = load_library()
        raise SqaError(status, f"{lib.sqa_status_string(status).decode()}: {lib.sqa_last_error().decode()}")


def _stream(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t, name, shape, dtype):
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def shape_of(q, k) -> Shape:
    B, N, Hq, dh = q.shape
    Hkv = k.shape[2]
    return Shape(B, N, Hq, Hkv, dh)


def fwd_workspace_bytes(B: int, N: int, H_q: int, H_kv: int, dh: int, causal: bool) -> int:
    return int(load_library().sqa_fwd_workspace_bytes(Shape(B, N, H_q, H_kv, dh), int(bool(causal))))


def sqa_fwd(q, k, v, out=None, lse=None, causal: bool = False, scale: float = 0.0, stream=None, workspace=None,
            key_ranges: bool = True):
    """Forward.  q [B,N,H_q,dh], k/v [B,N,H_kv,dh] bf16 CUDA tensors.
    Returns (out [B,N,H_q,dh] bf16, lse [B,H_q,N] fp32).  scale <= 0 means 1/sqrt(dh).
    Small problems split each Q tile's keys into ranges over several CTAs when
    key_ranges is true (sqa_fwd_with_workspace); workspace: a uint8 CUDA tensor
    of at least fwd_workspace_bytes(...) bytes, or None to allocate one."""
    import torch

    lib = load_library()
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q, k, v must be 4-D [B, N, H, dh]")
    s = shape_of(q, k)
    _need(q, "q", (s.B, s.N, s.H_q, s.dh), torch.bfloat16)
    _need(k, "k", (s.B, s.N, s.H_kv, s.dh), torch.bfloat16)
    _need(v, "v", (s.B, s.N, s.H_kv, s.dh), torch.bfloat16)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((s.B, s.H_q, s.N), dtype=torch.float32, device=q.device)
    _need(out, "out", (s.B, s.N, s.H_q, s.dh), torch.bfloat16)
    _need(lse, "lse", (s.B, s.H_q, s.N), torch.float32)
    need = int(lib.sqa_fwd_workspace_bytes(s, int(bool(causal)))) if key_ranges else 0
    if need == 0:
        _check(lib.sqa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), s,
                           int(bool(causal)), float(scale), _stream(stream)))
        return out, lse
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace.dtype != torch.uint8 or not workspace.is_cuda or workspace.numel() < need:
        raise ValueError(f"workspace must be a uint8 CUDA tensor of at least {need} bytes")
    _check(lib.sqa_fwd_with_workspace(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                      workspace.data_ptr(), workspace.numel(), s, int(bool(causal)),
                                      float(scale), _stream(stream)))
    return out, lse


def decode_workspace_bytes(B: int, N: int, H_q: int, H_kv: int, dh: int) -> int:
    return int(load_library().sqa_decode_workspace_bytes(Shape(B, N, H_q, H_kv, dh)))


def sqa_decode(q, k_cache, v_cache, seq_lens=None, out=None, lse=None, workspace=None, scale: float = 0.0,
               stream=None):
    """Decoding step.  q [B,H_q,dh] bf16 (one token per sequence), k_cache/v_cache
    [B,N,H_kv,dh] bf16, seq_lens int32 [B] on the device (None: all N).
    Returns (out [B,H_q,dh] bf16, lse [B,H_q] fp32)."""
    import torch

    lib = load_library()
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B, H_q, dh] and the caches [B, N, H_kv, dh]")
    B, Hq, dh = q.shape
    N, Hkv = k_cache.shape[1], k_cache.shape[2]
    s = Shape(B, N, Hq, Hkv, dh)
    _need(q, "q", (B, Hq, dh), torch.bfloat16)
    _need(k_cache, "k_cache", (B, N, Hkv, dh), torch.bfloat16)
    _need(v_cache, "v_cache", (B, N, Hkv, dh), torch.bfloat16)
    if seq_lens is not None:
        _need(seq_lens, "seq_lens", (B,), torch.int32)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    _need(out, "out", (B, Hq, dh), torch.bfloat16)
    _need(lse, "lse", (B, Hq), torch.float32)
    need = int(lib.sqa_decode_workspace_bytes(s))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib.sqa_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                          0 if seq_lens is None else seq_lens.data_ptr(), out.data_ptr(), lse.data_ptr(),
                          workspace.data_ptr(), workspace.numel() * workspace.element_size(), s, float(scale),
                          _stream(stream)))
    return out, lse


def bwd_workspace_bytes(B: int, N: int, H_q: int, H_kv: int, dh: int) -> int:
    return int(load_library().sqa_bwd_workspace_bytes(Shape(B, N, H_q, H_kv, dh)))


def sqa_bwd(dout, q, k, v, out, lse, dq=None, dk=None, dv=None, workspace=None, causal: bool = False,
            scale: float = 0.0, stream=None):
    """Backward of sum(dout * out).  Returns (dq, dk, dv) as bf16 CUDA tensors."""
    import torch

    lib = load_library()
    s = shape_of(q, k)
    _need(q, "q", (s.B, s.N, s.H_q, s.dh), torch.bfloat16)
    _need(k, "k", (s.B, s.N, s.H_kv, s.dh), torch.bfloat16)
    _need(v, "v", (s.B, s.N, s.H_kv, s.dh), torch.bfloat16)
    _need(dout, "dout", (s.B, s.N, s.H_q, s.dh), torch.bfloat16)
    _need(out, "out", (s.B, s.N, s.H_q, s.dh), torch.bfloat16)
    _need(lse, "lse", (s.B, s.H_q, s.N), torch.float32)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _need(dq, "dq", (s.B, s.N, s.H_q, s.dh), torch.bfloat16)
    _need(dk, "dk", (s.B, s.N, s.H_kv, s.dh), torch.bfloat16)
    _need(dv, "dv", (s.B, s.N, s.H_kv, s.dh), torch.bfloat16)
    need = int(lib.sqa_bwd_workspace_bytes(s))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check(lib.sqa_bwd(dout.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                       lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                       workspace.numel() * workspace.element_size(), s, int(bool(causal)), float(scale),
                       _stream(stream)))
    return dq, dk, dv


def set_timing_events(kernel: int, start=None, stop=None):
    """Record torch.cuda.Event `start`/`stop` around the main kernel of sqa_fwd
    (kernel=0) or sqa_bwd (kernel=1) on this thread; None turns it off."""
    lib = load_library()

    def handle(ev):
        if ev is None:
            return ctypes.c_void_p(None)
        if not ev.cuda_event:  # torch creates the CUDA event on its first record
            ev.record()
        return ctypes.c_void_p(ev.cuda_event)

    s, e = handle(start), handle(stop)
    _check(lib.sqa_set_timing_events(int(kernel), s, e))


def timeout_info(clear: bool = True):
    """First wait that gave up on this device: None, or a dict (block, role, barrier, thread, parity)."""
    lib = load_library()
    info = (ctypes.c_uint * 4)()
    _check(lib.sqa_device_timeout_info(info, int(bool(clear))))
    if info[0] == 0:
        return None
    return {"block": int(info[1]), "role": int(info[2] >> 16), "barrier": int(info[2] & 0xFFFF),
            "thread": int(info[3] >> 8), "parity": int(info[3] & 0xFF)}


def device_status(clear: bool = True) -> int:
    """Synchronise and return the device wait-status word (0 = no wait gave up)."""
    lib = load_library()
    w = ctypes.c_uint(0)
    _check(lib.sqa_device_status(ctypes.byref(w), int(bool(clear))))
    return int(w.value)


def layer_workspace_bytes(B: int, N: int, d: int, H_q: int, H_kv: int, dh: int, backward: bool) -> int:
    return int(load_library().sqa_layer_workspace_bytes(LayerShape(B, N, d, H_q, H_kv, dh), int(bool(backward))))


def _layer_shape(x, w_qkv, w_o, H_q, H_kv):
    import torch

    if x.dim() != 3:
        raise ValueError("x must be [B, N, d]")
    B, N, d = x.shape
    dh = w_o.shape[0] // H_q
    s = LayerShape(B, N, d, H_q, H_kv, dh)
    _need(x, "x", (B, N, d), torch.bfloat16)
    _need(w_qkv, "w_qkv", (d, (H_q + 2 * H_kv) * dh), torch.bfloat16)
    _need(w_o, "w_o", (H_q * dh, d), torch.bfloat16)
    return s


def sqa_layer_fwd(x, w_qkv, w_o, H_q: int, H_kv: int, causal: bool = True, scale: float = 0.0,
                  rope_base: float = 10000.0, workspace=None, stream=None):
    """Layer forward.  x [B,N,d], w_qkv [d,(H_q+2H_kv)dh], w_o [H_q dh,d] (bf16 CUDA).
    Returns (y, saved) with saved = dict(q, k, v, out, lse) for sqa_layer_bwd."""
    import torch

    lib = load_library()
    s = _layer_shape(x, w_qkv, w_o, H_q, H_kv)
    dev = x.device
    y = torch.empty_like(x)
    q = torch.empty((s.B, s.N, H_q, s.dh), dtype=torch.bfloat16, device=dev)
    k = torch.empty((s.B, s.N, H_kv, s.dh), dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)
    out = torch.empty_like(q)
    lse = torch.empty((s.B, H_q, s.N), dtype=torch.float32, device=dev)
    need = int(lib.sqa_layer_workspace_bytes(s, 0))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib.sqa_layer_fwd(x.data_ptr(), w_qkv.data_ptr(), w_o.data_ptr(), y.data_ptr(), q.data_ptr(),
                             k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), s, int(bool(causal)), float(scale),
                             float(rope_base), _stream(stream)))
    return y, {"q": q, "k": k, "v": v, "out": out, "lse": lse}


def sqa_layer_bwd(dy, x, w_qkv, w_o, saved, H_q: int, H_kv: int, causal: bool = True, scale: float = 0.0,
                  rope_base: float = 10000.0, workspace=None, stream=None):
    """Layer backward of sum(dy * y).  Returns (dx bf16, dw_qkv fp32, dw_o fp32)."""
    import torch

    lib = load_library()
    s = _layer_shape(x, w_qkv, w_o, H_q, H_kv)
    _need(dy, "dy", tuple(x.shape), torch.bfloat16)
    dev = x.device
    dx = torch.empty_like(x)
    dw_qkv = torch.empty(tuple(w_qkv.shape), dtype=torch.float32, device=dev)
    dw_o = torch.empty(tuple(w_o.shape), dtype=torch.float32, device=dev)
    need = int(lib.sqa_layer_workspace_bytes(s, 1))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    sv = saved
    _check(lib.sqa_layer_bwd(dy.data_ptr(), x.data_ptr(), w_qkv.data_ptr(), w_o.data_ptr(), sv["q"].data_ptr(),
                             sv["k"].data_ptr(), sv["v"].data_ptr(), sv["out"].data_ptr(), sv["lse"].data_ptr(),
                             dx.data_ptr(), dw_qkv.data_ptr(), dw_o.data_ptr(), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), s, int(bool(causal)), float(scale),
                             float(rope_base), _stream(stream)))
    return dx, dw_qkv, dw_o


class BlockShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int), ("H_q", ctypes.c_int),
                ("H_kv", ctypes.c_int), ("dh", ctypes.c_int), ("hidden", ctypes.c_int)]


_BLOCK_PARAMS = ("g1", "w_qkv", "w_o", "g2", "w1", "w3", "w2")


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _BLOCK_PARAMS]


class BlockGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _BLOCK_PARAMS]


def _block_lib():
    lib = load_library()
    if not getattr(lib, "_block_bound", False):
        vp, sz, c_int, c_float = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
        lib.sqa_block_state_bytes.argtypes = [BlockShape]
        lib.sqa_block_state_bytes.restype = sz
        lib.sqa_block_fwd.argtypes = [vp, ctypes.POINTER(BlockWeights), vp, vp, sz, BlockShape, c_int, c_float,
                                      c_float, vp]
        lib.sqa_block_fwd.restype = c_int
        lib.sqa_block_bwd.argtypes = [vp, vp, ctypes.POINTER(BlockWeights), vp, sz, vp, ctypes.POINTER(BlockGrads),
                                      BlockShape, c_int, c_float, c_float, vp]
        lib.sqa_block_bwd.restype = c_int
        lib._block_bound = True
    return lib


def _block_shape(x, w, H_q, H_kv):
    import torch

    if x.dim() != 3:
        raise ValueError("x must be [B, N, d]")
    B, N, d = x.shape
    dh = w["w_o"].shape[0] // H_q
    hidden = w["w1"].shape[1]
    shapes = {"g1": (d,), "w_qkv": (d, (H_q + 2 * H_kv) * dh), "w_o": (H_q * dh, d), "g2": (d,),
              "w1": (d, hidden), "w3": (d, hidden), "w2": (hidden, d)}
    _need(x, "x", (B, N, d), torch.bfloat16)
    for n in _BLOCK_PARAMS:
        _need(w[n], n, shapes[n], torch.bfloat16)
    return BlockShape(B, N, d, H_q, H_kv, dh, hidden), shapes


def block_state_bytes(B, N, d, H_q, H_kv, dh, hidden) -> int:
    return int(_block_lib().sqa_block_state_bytes(BlockShape(B, N, d, H_q, H_kv, dh, hidden)))


def sqa_block_fwd(x, weights: dict, H_q: int, H_kv: int, state=None, causal: bool = True, scale: float = 0.0,
                  rope_base: float = 10000.0, stream=None):
    """One SQAT-m block forward.  weights: dict of bf16 CUDA tensors g1, w_qkv,
    w_o, g2, w1, w3, w2.  Returns (y, state); pass state to sqa_block_bwd."""
    import torch

    lib = _block_lib()
    s, _ = _block_shape(x, weights, H_q, H_kv)
    if state is None:
        state = torch.empty(max(int(lib.sqa_block_state_bytes(s)), 256), dtype=torch.uint8, device=x.device)
    y = torch.empty_like(x)
    w = BlockWeights(*(weights[n].data_ptr() for n in _BLOCK_PARAMS))
    _check(lib.sqa_block_fwd(x.data_ptr(), ctypes.byref(w), y.data_ptr(), state.data_ptr(),
                             state.numel() * state.element_size(), s, int(bool(causal)), float(scale),
                             float(rope_base), _stream(stream)))
    return y, state


def sqa_block_bwd(dy, x, weights: dict, state, H_q: int, H_kv: int, causal: bool = True, scale: float = 0.0,
                  rope_base: float = 10000.0, stream=None):
    """Block backward of sum(dy * y).  Returns (dx bf16, dict of fp32 gradients)."""
    import torch

    lib = _block_lib()
    s, shapes = _block_shape(x, weights, H_q, H_kv)
    _need(dy, "dy", tuple(x.shape), torch.bfloat16)
    dx = torch.empty_like(x)
    grads = {n: torch.empty(shapes[n], dtype=torch.float32, device=x.device) for n in _BLOCK_PARAMS}
    w = BlockWeights(*(weights[n].data_ptr() for n in _BLOCK_PARAMS))
    gr = BlockGrads(*(grads[n].data_ptr() for n in _BLOCK_PARAMS))
    _check(lib.sqa_block_bwd(dy.data_ptr(), x.data_ptr(), ctypes.byref(w), state.data_ptr(),
                             state.numel() * state.element_size(), dx.data_ptr(), ctypes.byref(gr), s,
                             int(bool(causal)), float(scale), float(rope_base), _stream(stream)))
    return dx, grads
