"""Seeded synthetic inputs for Sparse Query Attention workloads.

This module only draws random tensors and names workload shapes; it holds
none of the attention arithmetic.  The CUDA path's tests, the benchmark and
the oracle-side tests all take their inputs from here, so both sides see the
same bf16 bits.

Recipe: a CPU ``torch.Generator`` seeded with ``seed`` draws standard normal
fp32 tensors in the order q, k, v, dO; each is multiplied by its standard
deviation (and K by ``k_scale``) and then rounded to bf16.  Shapes follow the
SQAT-m model card ("Architecture details": d = 256 split over 16 heads, so
dh = 16; 8 query groups and 4 key/value groups; message length 1024) and the
arXiv 2510.01817 abstract (32k-200k token sequences), plus a larger-model
dh = 128 case.  The pages train on Wikipedia text; attention inputs here are
synthetic Gaussians instead, since the attention core needs no tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    Hq: int
    Hkv: int
    dh: int
    causal: bool
    backward: bool
    std: float = 1.0
    k_scale: float = 1.0
    scale: float = 0.0  # <= 0 selects 1/sqrt(dh)
    note: str = ""
    decode: bool = False  # one new query token per sequence against a cache of N positions
    d: int = 0            # decoder-block stacks: model width, SwiGLU width, number of blocks
    hidden: int = 0
    layers: int = 0
    graph: bool = False   # launch-bound: the benchmark replays each step as a CUDA graph

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale > 0 else self.dh ** -0.5

    @property
    def block(self) -> bool:
        return self.layers > 0


# Workload shapes.  Each is one (B, N, H_q, H_kv, dh) point; sweeps list one
# entry per head configuration.
WORKLOADS: dict[str, Workload] = {}


def _add(w: Workload):
    WORKLOADS[w.name] = w


# SQAT-m single-layer attention, forward only.
_add(Workload("sqatm_layer_fwd", 1, 1024, 8, 4, 16, True, False, scale=0.25, graph=True,
              note="SQAT-m single layer, B=1 N=1024 dh=16 Hq=8 Hkv=4 causal"))
# SQAT-m training-step attention (forward + backward) and its same-kernel comparisons.
for hq, hkv, tag in ((8, 4, "sqa"), (16, 4, "gqa"), (16, 16, "mha"), (16, 1, "mqa")):
    _add(Workload(f"sqatm_train_{tag}", 32, 1024, hq, hkv, 16, True, True,
                  note=f"SQAT-m training step, B=32 N=1024 dh=16 Hq={hq} Hkv={hkv} causal"))
# Long-context encoder attention, N=32768, head sweep.
for hq, hkv in ((8, 4), (8, 8), (4, 4), (16, 16), (16, 4), (16, 1)):
    _add(Workload(f"enc32k_{hq}_{hkv}", 1, 32768, hq, hkv, 16, False, False,
                  note=f"encoder, B=1 N=32768 dh=16 Hq={hq} Hkv={hkv} bidirectional"))
# Long-context encoder attention at 131072 and 200000 tokens (200000 is not a tile multiple).
for n in (131072, 200000):
    for hq, hkv in ((4, 4), (8, 4)):
        _add(Workload(f"enc{n // 1000}k_{hq}_{hkv}", 1, n, hq, hkv, 16, False, False, std=0.5,
                      note=f"encoder, B=1 N={n} dh=16 Hq={hq} Hkv={hkv} bidirectional, std 0.5"))
# Larger-model SQA: d=2048 over 16 heads, dh=128; the same kernel with every
# head kept (MHA 16/16), GQA 16/4 and MQA 16/1 for comparison.
_add(Workload("large_dh128", 2, 65536, 8, 4, 128, True, True, k_scale=0.1,
              note="larger model, B=2 N=65536 dh=128 Hq=8 Hkv=4 causal, K x 0.1"))
for hq, hkv, tag in ((16, 16, "mha"), (16, 4, "gqa"), (16, 1, "mqa")):
    _add(Workload(f"large_dh128_{tag}", 2, 65536, hq, hkv, 128, True, True, k_scale=0.1,
                  note=f"larger model, B=2 N=65536 dh=128 Hq={hq} Hkv={hkv} causal, K x 0.1"))
# The same head layout at 16384 tokens, small enough for full profiler captures.
_add(Workload("large_dh128_16k", 1, 16384, 8, 4, 128, True, True, k_scale=0.1,
              note="larger model, B=1 N=16384 dh=128 Hq=8 Hkv=4 causal, K x 0.1"))
# SQAT-m decoder-block stack (RMSNorm, the SQA layer with its projections and
# the rotary embedding, SwiGLU 768; 8 blocks, d = 256, dh = 16, causal), one
# forward and backward step with random weights (SQAT-m card, "Architecture
# details"; its "Time per batch" table compares whole-model steps of the head
# layouts), with the same comparisons as the training-step attention.
for hq, hkv, tag in ((8, 4, "sqa"), (16, 4, "gqa"), (16, 16, "mha"), (16, 1, "mqa")):
    _add(Workload(f"sqatm_block_{tag}", 32, 1024, hq, hkv, 16, True, True, d=256, hidden=768, layers=8, graph=True,
                  note=f"SQAT-m 8-block stack, B=32 N=1024 d=256 dh=16 Hq={hq} Hkv={hkv} SwiGLU 768 causal"))
# Decoding step: a batch of sequences, each adding one token against a full
# key/value cache (SQAT-m head layout, and the larger-model dh=128 layout).
_add(Workload("decode_sqatm", 32, 32768, 8, 4, 16, False, False, decode=True,
              note="decode step, B=32 sequences, cache N=32768, dh=16 Hq=8 Hkv=4"))
_add(Workload("decode_dh128", 8, 65536, 8, 4, 128, False, False, k_scale=0.1, decode=True,
              note="decode step, B=8 sequences, cache N=65536, dh=128 Hq=8 Hkv=4, K x 0.1"))
# MQA head layout (16 query heads on one K/V head): a group of 16 takes the
# shared-memory split path.
_add(Workload("decode_mqa", 32, 32768, 16, 1, 16, False, False, decode=True,
              note="decode step, B=32 sequences, cache N=32768, dh=16 Hq=16 Hkv=1"))


def make_inputs(B: int, N: int, Hq: int, Hkv: int, dh: int, seed: int = 0, std: float = 1.0,
                k_scale: float = 1.0, with_dout: bool = False):
    """Draw q [B,N,Hq,dh], k, v [B,N,Hkv,dh] (and dO [B,N,Hq,dh]) as CPU bf16 tensors."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    q = (torch.randn(B, N, Hq, dh, generator=g) * std).to(torch.bfloat16)
    k = (torch.randn(B, N, Hkv, dh, generator=g) * (std * k_scale)).to(torch.bfloat16)
    v = (torch.randn(B, N, Hkv, dh, generator=g) * std).to(torch.bfloat16)
    dout = torch.randn(B, N, Hq, dh, generator=g).to(torch.bfloat16) if with_dout else None
    return q, k, v, dout


def make_decode_inputs(B: int, N: int, Hq: int, Hkv: int, dh: int, seed: int = 0, std: float = 1.0,
                       k_scale: float = 1.0):
    """Draw the new token's queries q [B,Hq,dh] and the caches k, v [B,N,Hkv,dh] (CPU bf16), in that order."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    q = (torch.randn(B, Hq, dh, generator=g) * std).to(torch.bfloat16)
    k = (torch.randn(B, N, Hkv, dh, generator=g) * (std * k_scale)).to(torch.bfloat16)
    v = (torch.randn(B, N, Hkv, dh, generator=g) * std).to(torch.bfloat16)
    return q, k, v


def workload_inputs(w: Workload, seed: int = 0):
    """(q, k, v, dout); for a decoding workload q is [B,Hq,dh] and dout is None;
    for a block stack (x, weights, dy, None) from make_block_inputs."""
    if w.block:
        return (*make_block_inputs(w.B, w.N, w.d, w.Hq, w.Hkv, w.dh, w.hidden, seed=seed), None)
    if w.decode:
        return (*make_decode_inputs(w.B, w.N, w.Hq, w.Hkv, w.dh, seed=seed, std=w.std, k_scale=w.k_scale), None)
    return make_inputs(w.B, w.N, w.Hq, w.Hkv, w.dh, seed=seed, std=w.std, k_scale=w.k_scale,
                       with_dout=w.backward)


def make_layer_inputs(B: int, N: int, d: int, Hq: int, Hkv: int, dh: int, seed: int = 0):
    """Draw x [B,N,d], the fused projection w_qkv [d, (Hq + 2 Hkv) dh], w_o
    [Hq dh, d] and the upstream gradient dy [B,N,d] (CPU bf16), in that order.
    x and dy are standard normal; each weight has standard deviation
    1/sqrt(fan-in), so the projections keep unit variance."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    x = torch.randn(B, N, d, generator=g).to(torch.bfloat16)
    w_qkv = (torch.randn(d, (Hq + 2 * Hkv) * dh, generator=g) * d ** -0.5).to(torch.bfloat16)
    w_o = (torch.randn(Hq * dh, d, generator=g) * (Hq * dh) ** -0.5).to(torch.bfloat16)
    dy = torch.randn(B, N, d, generator=g).to(torch.bfloat16)
    return x, w_qkv, w_o, dy


def make_block_inputs(B: int, N: int, d: int, Hq: int, Hkv: int, dh: int, hidden: int, seed: int = 0):
    """Draw x [B,N,d], the block's weights and dy [B,N,d] (CPU bf16), in the
    order x, g1, w_qkv, w_o, g2, w1, w3, w2, dy.  The norm gains are 1 + 0.1
    N(0,1); each matrix has standard deviation 1/sqrt(fan-in)."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))

    def mat(rows, cols):
        return (torch.randn(rows, cols, generator=g) * rows ** -0.5).to(torch.bfloat16)

    x = torch.randn(B, N, d, generator=g).to(torch.bfloat16)
    w = {"g1": (1.0 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16),
         "w_qkv": mat(d, (Hq + 2 * Hkv) * dh), "w_o": mat(Hq * dh, d),
         "g2": (1.0 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16),
         "w1": mat(d, hidden), "w3": mat(d, hidden), "w2": mat(hidden, d)}
    dy = torch.randn(B, N, d, generator=g).to(torch.bfloat16)
    return x, w, dy
