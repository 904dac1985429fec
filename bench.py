#!/usr/bin/env python
"""Benchmark of the Sparse Query Attention hot path on B200.

One step is one pass of the whole path over one batch: sqa_fwd followed by
sqa_bwd (for forward-only workloads, sqa_fwd alone).  The default workload is
the largest single-GPU configuration: larger-model SQA attention, B=2,
N=65536, dh=128 (d=2048 split over 16 heads), H_q=8 query heads over H_kv=4
key/value heads, causal, forward and backward, K scaled by 0.1 (arXiv
2510.01817 abstract: the gains are claimed for 32k-200k token sequences).
After it the same kernels run the MHA (16/16), GQA (16/4) and MQA (16/1) head
layouts of the same model for comparison (``--no-compare`` skips them); the
SQAT-m training step (B=32, N=1024, dh=16, 8/4) and the other shapes are
available with ``--workload``.

Throughput counts 4*B*H_q*N^2*dh FLOPs for the forward (halved when causal)
and 3.5 times that for forward plus backward.  Inputs are seeded synthetic bf16
Gaussians; several buffer sets whose total exceeds the 126 MB L2 are used in
rotation, so every step reads its inputs from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--no-compare]
  python bench.py --impl reference ...   # the fp64 CPU oracle on a bounded sample

Without --steps the number of timed steps follows from the warm-up's step time:
about 20 s of timed work for the workload (at least 5 steps, at most 2000) and
about 8 s for each comparison layout, so a run without flags ends within a few
minutes; with --steps K exactly K steps are timed, comparisons included.

Under torchrun every rank runs its own copy of the workload (independent
batches, no collective on the data path): weak scaling.  One JSON line is
printed by rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
SM_COUNT = 148
SM_MAX_MHZ = 1965.0
# Special-function unit: 16 exp2 results per clock per SM (4 per sub-partition).
SFU_EXP2_PER_CLK_PER_SM = 16


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about 20 s of the workload's warm-up step time)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_dh128")
    ap.add_argument("--no-compare", action="store_true",
                    help="skip the same-kernel MHA/GQA/MQA comparison after the workload")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="time budget of the CPU-baseline sample")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--shard", action="store_true",
                    help="under torchrun: split one problem over the ranks by (batch entry, KV head) "
                         "(strong scaling) instead of a replica per rank")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step from the host even where the workload asks for CUDA-graph replay")
    return ap.parse_args()


def block_gemm_params(w) -> int:
    """Weights of one decoder block's matrix products: W_q|W_k|W_v, W_o, W1, W3, W2."""
    return w.d * (w.Hq + 2 * w.Hkv) * w.dh + w.Hq * w.dh * w.d + 3 * w.d * w.hidden


def counted_flops(w) -> float:
    if w.decode:  # one query row per (sequence, head) against N cached positions
        return 4.0 * w.B * w.Hq * w.N * w.dh
    fwd = 4.0 * w.B * w.Hq * w.N * w.N * w.dh
    if w.causal:
        fwd /= 2
    attn = fwd * (3.5 if w.backward else 1.0)
    if w.block:  # per block: the attention plus its matrix products (forward once, backward twice)
        return w.layers * (attn + 2.0 * w.B * w.N * block_gemm_params(w) * (3.0 if w.backward else 1.0))
    return attn


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' values, returned on every rank (x itself on one rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(w, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the work of every rank's replica over the slowest rank's step time."""
    return counted_flops(w) * world / (ms_per_step * 1e-3) / 1e12


def score_elements(w) -> float:
    """Unmasked (query row, key) pairs over all query heads: one exp2 each."""
    if w.decode:
        return float(w.B) * w.Hq * w.N
    per = w.N * (w.N + 1) / 2 if w.causal else float(w.N) * w.N
    return w.B * w.Hq * per


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# --------------------------------------------------------------------------- CPU oracle
def oracle_subproblem(w, seed=0):
    """One independent slice of the workload: batch entry 0, KV head 0 and its
    g query heads (the oracle's work on it scales with the counted FLOPs); for
    a block stack, one block of batch entry 0."""
    from sparse_query_attention_sqa_b200.inputs import make_block_inputs, make_decode_inputs, make_inputs

    if w.block:
        x, wd, dy = make_block_inputs(1, w.N, w.d, w.Hq, w.Hkv, w.dh, w.hidden, seed=seed)
        sub = type(w)(name=w.name + "_slice", B=1, N=w.N, Hq=w.Hq, Hkv=w.Hkv, dh=w.dh, causal=w.causal,
                      backward=w.backward, d=w.d, hidden=w.hidden, layers=1)
        # the oracle block takes fp64 arrays and the fused projection split into W_q, W_k, W_v
        wf = {n: t.double().numpy() for n, t in wd.items()}
        nq, nk = w.Hq * w.dh, w.Hkv * w.dh
        p = {"g1": wf["g1"], "g2": wf["g2"], "wq": wf["w_qkv"][:, :nq], "wk": wf["w_qkv"][:, nq:nq + nk],
             "wv": wf["w_qkv"][:, nq + nk:], "wo": wf["w_o"], "w1": wf["w1"], "w3": wf["w3"], "w2": wf["w2"]}
        return sub, (x.double().numpy(), p, dy.double().numpy(), None)
    g = w.Hq // w.Hkv
    if w.decode:
        q, k, v = make_decode_inputs(1, w.N, g, 1, w.dh, seed=seed, std=w.std, k_scale=w.k_scale)
        dout = None
    else:
        q, k, v, dout = make_inputs(1, w.N, g, 1, w.dh, seed=seed, std=w.std, k_scale=w.k_scale,
                                    with_dout=w.backward)
    sub = type(w)(name=w.name + "_slice", B=1, N=w.N, Hq=g, Hkv=1, dh=w.dh, causal=w.causal, backward=w.backward,
                  std=w.std, k_scale=w.k_scale, scale=w.scale, decode=w.decode)
    return sub, (q, k, v, dout)


def run_oracle_step(sub, data):
    import oracle

    if sub.block:
        from oracle import block as oblock

        x, wd, dy, _ = data
        oblock.block_fwd(x, wd, sub.Hq, sub.Hkv, sub.causal)
        if sub.backward:
            oblock.block_bwd(x, wd, dy, sub.Hq, sub.Hkv, sub.causal)
        return
    q, k, v, dout = data
    if sub.decode:
        oracle.sqa_decode(q, k, v, None, sub.softmax_scale)
        return
    oracle.sqa_fwd(q, k, v, sub.causal, sub.softmax_scale)
    if sub.backward:
        oracle.sqa_bwd(q, k, v, dout, sub.causal, sub.softmax_scale)


def omp_threads() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def cpu_baseline_rows(w, seconds):
    """For workloads where one slice is too long for the budget: forward rows."""
    import numpy as np

    import oracle
    from sparse_query_attention_sqa_b200.inputs import workload_inputs

    q, k, v, _ = workload_inputs(w)
    rng = np.random.default_rng(0)
    n_rows, t_total, flops, done = 8, 0.0, 0.0, 0
    while t_total < seconds:
        rows = rng.integers(0, w.N, n_rows)
        trip = np.stack([np.zeros_like(rows), rows, rng.integers(0, w.Hq, n_rows)], 1)
        t = time.perf_counter()
        oracle.sqa_fwd_rows(q[:1], k[:1], v[:1], trip, w.causal, w.softmax_scale)
        t_total += time.perf_counter() - t
        flops += sum(4.0 * w.dh * ((int(i) + 1) if w.causal else w.N) for i in rows)
        done += n_rows
    return {"value": flops / t_total / 1e12, "unit": "TFLOP/s", "cores": omp_threads(), "kind": "oracle",
            "sample": f"fp64 oracle forward of {done} random query rows of batch entry 0 (N={w.N}, dh={w.dh}) "
                      f"in {t_total:.1f} s; forward FLOPs only"}


def cpu_baseline(w, seconds):
    g = w.Hq // w.Hkv
    if not w.decode and not w.block and g * w.N * w.N * w.dh > 2 ** 34:  # one slice would take minutes
        return cpu_baseline_rows(w, seconds)
    sub, data = oracle_subproblem(w)
    run_oracle_step(sub, data)  # builds the oracle and warms caches
    t0 = time.perf_counter()
    n = 0
    while True:
        run_oracle_step(sub, data)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    rate = counted_flops(sub) * n / el / 1e12
    what = (f"one decoder block of batch entry 0 (N={w.N}, d={w.d})" if w.block else
            f"batch entry 0, KV head 0 and its {sub.Hq} query heads (N={w.N}, dh={w.dh})")
    return {"value": rate, "unit": "TFLOP/s", "cores": omp_threads(), "kind": "oracle",
            "sample": f"fp64 oracle {pass_name(w)} on {what}, {n} runs in {el:.1f} s"}


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, enabled, index):
        self.proc = None
        # Raw samples go to SQA_BENCH_CLOCKS_DIR (a temporary directory by default);
        # the JSON line carries their summary.
        import tempfile

        out_dir = os.environ.get("SQA_BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_bench_{os.getpid()}.csv")
        if not enabled:
            return
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(index),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------- GPU arm
BLOCK_PARAMS = ("g1", "w_qkv", "w_o", "g2", "w1", "w3", "w2")


def alloc_set(w, q, k, v, dout, lib, torch):
    dev = "cuda"
    if w.block:  # q, k, v are x, the weights, dy
        s = {"x": q.to(dev), "dy": v.to(dev)}
        s.update({"w_" + n: k[n].to(dev) for n in BLOCK_PARAMS})
        nbytes = max(lib.block_state_bytes(w.B, w.N, w.d, w.Hq, w.Hkv, w.dh, w.hidden), 256)
        for layer in range(w.layers):
            s[f"state{layer}"] = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        s["y"] = torch.empty_like(s["x"])
        s["dx"] = torch.empty_like(s["x"])
        return s
    s = {"q": q.to(dev), "k": k.to(dev), "v": v.to(dev)}
    s["out"] = torch.empty_like(s["q"])
    if w.decode:
        s["lse"] = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
        s["ws"] = torch.empty(lib.decode_workspace_bytes(w.B, w.N, w.Hq, w.Hkv, w.dh), dtype=torch.uint8,
                              device=dev)
        return s
    s["lse"] = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    fws = lib.fwd_workspace_bytes(w.B, w.N, w.Hq, w.Hkv, w.dh, w.causal)
    if fws > 0:  # small problems: the forward splits key ranges over CTAs
        s["fws"] = torch.empty(fws, dtype=torch.uint8, device=dev)
    if w.backward:
        s["dout"] = dout.to(dev)
        s["dq"] = torch.empty_like(s["q"])
        s["dk"] = torch.empty_like(s["k"])
        s["dv"] = torch.empty_like(s["v"])
        s["ws"] = torch.empty(lib.bwd_workspace_bytes(w.B, w.N, w.Hq, w.Hkv, w.dh), dtype=torch.uint8, device=dev)
    return s


def set_bytes(s) -> int:
    return sum(t.numel() * t.element_size() for t in s.values())


def step(lib, w, s):
    if w.block:
        # every block runs with the same random weights (a timing stack); the
        # weight gradients of each block are produced and dropped
        wd = {n: s["w_" + n] for n in BLOCK_PARAMS}
        xs = [s["x"]]
        for layer in range(w.layers):
            y, _ = lib.sqa_block_fwd(xs[-1], wd, w.Hq, w.Hkv, state=s[f"state{layer}"], causal=w.causal)
            xs.append(y)
        g = s["dy"]
        for layer in reversed(range(w.layers)):
            g, _ = lib.sqa_block_bwd(g, xs[layer], wd, s[f"state{layer}"], w.Hq, w.Hkv, causal=w.causal)
        s["y"], s["dx"] = xs[-1], g
        return
    if w.decode:
        lib.sqa_decode(s["q"], s["k"], s["v"], out=s["out"], lse=s["lse"], workspace=s["ws"], scale=w.scale)
        return
    lib.sqa_fwd(s["q"], s["k"], s["v"], out=s["out"], lse=s["lse"], causal=w.causal, scale=w.scale,
                workspace=s.get("fws"))
    if w.backward:
        lib.sqa_bwd(s["dout"], s["q"], s["k"], s["v"], s["out"], s["lse"], dq=s["dq"], dk=s["dk"], dv=s["dv"],
                    workspace=s["ws"], causal=w.causal, scale=w.scale)


def metric_name(w) -> str:
    return "SQAT-m decoder-block stack" if w.block else "SQA attention"


def launches_per_step(w) -> int:
    """Kernels of this library launched per step (memsets not counted)."""
    if w.block:
        # forward: RMSNorm, rotary table, W_qkv, attention, W_o, RMSNorm, W1|W3, W2;
        # backward: dM (SwiGLU), dW2, dW1, dW3, dN, RMSNorm; the layer (rotary
        # table, dO, dW_o, attention preprocess / main / dQ, two inverse
        # rotations, three dW_qkv parts, dX); RMSNorm
        return w.layers * (8 + 6 + 12 + 1)
    # the forward, the backward's preprocess, its main kernel and either the dQ
    # conversion (dh <= 32) or the dQ kernel (dh 64 / 128)
    return 4 if w.backward else (2 if w.decode else 1)


def pass_name(w) -> str:
    if w.block:
        return f"{w.layers}-block fwd+bwd"
    return "decode" if w.decode else ("fwd+bwd" if w.backward else "fwd")


def decode_bytes(w) -> float:
    """Algorithmic bytes of one decoding step: the whole K and V caches once,
    the new queries, the outputs and their lse."""
    return 2.0 * w.B * w.N * w.Hkv * w.dh * 2 + 2.0 * w.B * w.Hq * w.dh * 2 + 4.0 * w.B * w.Hq


def launched_kernel(w, hook: int) -> str:
    """Name (with template arguments) of the main kernel behind a timing hook:
    0 the forward, 1 the backward, 2 the decoding split kernel."""
    if hook == 0:
        return f"sqa_fwd_kernel<{w.dh}>"
    g = w.Hq // w.Hkv
    if hook == 1:  # at dh 64 / 128 the hook brackets the dK/dV and the dQ kernels
        if w.dh <= 32:
            return f"sqa_bwd_tf32_kernel<{w.dh}>"
        lo = "true" if g >= 6 else "false"  # groups of 6+ carry P and dS as bf16 hi + lo
        return f"sqa_bwd_kernel<{w.dh},{lo}>+sqa_bwd_q_kernel<{w.dh}>"
    if g <= 4 and (w.Hkv & (w.Hkv - 1)) == 0 and w.Hkv <= 2048 // w.dh:  # register-resident path
        return f"sqa_decode_split_kernel<{w.dh},{g}>"
    if 5 <= g <= 16:  # tensor-core path
        return f"sqa_decode_mma_kernel<{w.dh}>"
    return f"sqa_decode_split_kernel<{w.dh},0>"


def roofline_for(w, kernel_name, ms, peaks, peak_kind):
    if w.decode:
        # HBM-bound: stream the caches once
        achieved = decode_bytes(w) / (ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic_for(kernel_name, w), "kernel": kernel_name, "peak_source": f"{peak_kind} hbm_gbs"}
    if w.dh <= 32:
        # exp-bound: one exp2 per unmasked score element on the special-function unit
        units = score_elements(w)
        achieved = units / (ms * 1e-3) / 1e9
        peak = SM_COUNT * SFU_EXP2_PER_CLK_PER_SM * SM_MAX_MHZ * 1e6 / 1e9
        return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Gexp2/s", "frac": achieved / peak,
                "traffic": traffic_for(kernel_name, w), "kernel": kernel_name,
                "peak_source": "derived: 148 SMs x 16 exp2/clk/SM x 1965 MHz"}
    flops = 4.0 * w.B * w.Hq * w.N * w.N * w.dh / (2 if w.causal else 1)
    if kernel_name.startswith("sqa_bwd"):
        flops *= 2.5
    achieved = flops / (ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained")
    rl = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
          "traffic": traffic_for(kernel_name, w), "kernel": kernel_name, "peak_source": f"{peak_kind} bf16_tflops"}
    if sustained:
        rl["peak_sustained"] = sustained
        rl["frac_sustained"] = achieved / sustained
    return rl


def strip_c_comments(text: str) -> str:
    """C/C++ source with its comments removed (string and character literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i : j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "".join(out)


def kernel_source_sha256():
    """Hash of the code (comments removed, whitespace runs collapsed) of every
    CUDA source of the library: a profile is valid only for the code it measured."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_query_attention_sqa_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, fn), encoding="utf-8") as f:
                code = " ".join(strip_c_comments(f.read()).split())  # layout ignored too
                h.update(fn.encode() + b"\0" + code.encode())
    return h.hexdigest()


def traffic_for(kernel_name, w):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except Exception:
        return None
    digest = kernel_source_sha256()
    for e in table.get("entries", []):
        if e.get("kernel") == kernel_name and e.get("workload") == w.name and e.get("source_sha256") == digest:
            return e.get("dram_bytes_per_launch")
    return None


class GraphSteps:
    """CUDA graphs holding whole steps, for launch-bound workloads (the step's
    launches cost the host more than the device's work).  A step of a single
    launch takes about as long on the device as the host needs to replay a
    graph, so such steps are captured `per_graph` at a time over consecutive
    buffer sets; run(k) replays exactly k steps.  The timing hooks are off
    while capturing."""

    def __init__(self, lib, w, sets, torch, per_graph):
        self.lib, self.w, self.sets, self.torch, self.per = lib, w, sets, torch, per_graph
        self.graphs = [self._capture(start, per_graph) for start in range(0, len(sets), per_graph)]
        self.tails = {}
        for gph in self.graphs:
            gph.replay()
        torch.cuda.synchronize()
        assert lib.device_status() == 0, "a kernel wait gave up in a graph's first replay"

    def _capture(self, start, count):
        gph = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(gph, capture_error_mode="thread_local"):
            for i in range(count):
                step(self.lib, self.w, self.sets[(start + i) % len(self.sets)])
        return gph

    def prepare(self, k):
        """Capture the graph of the last k % per_graph steps before timing."""
        rem = k % self.per
        if rem and rem not in self.tails:
            self.tails[rem] = self._capture(0, rem)
            self.tails[rem].replay()
            self.torch.cuda.synchronize()

    def run(self, k):
        full, rem = divmod(k, self.per)
        for i in range(full):
            self.graphs[i % len(self.graphs)].replay()
        if rem:
            self.tails[rem].replay()


def graph_steps(lib, w, sets, torch, args):
    if not w.graph or args.no_graph:
        return None
    return GraphSteps(lib, w, sets, torch, 16 if launches_per_step(w) == 1 else 1)


def warm_up(lib, w, sets, warmup, torch):
    """Warm-up steps; each times its main kernels with the library's hook.
    Returns ({kernel: [ms]}, the dominant kernel's name, its hook index, the
    median step time in ms)."""
    ev = lambda: torch.cuda.Event(enable_timing=True)
    kern, steps_ms = {}, []
    hooks = (2,) if w.decode else ((0, 1) if w.backward else (0,))  # timing-hook indices: fwd, bwd, decode
    for i in range(max(warmup, 3)):
        s = sets[i % len(sets)]
        evs = {h: (ev(), ev()) for h in hooks}
        for h, (e0, e1) in evs.items():
            lib.set_timing_events(h, e0, e1)
        a, b = ev(), ev()
        a.record()
        step(lib, w, s)
        b.record()
        for h in hooks:
            lib.set_timing_events(h)
        torch.cuda.synchronize()
        steps_ms.append(a.elapsed_time(b))
        for h, (e0, e1) in evs.items():
            kern.setdefault(launched_kernel(w, h), []).append(e0.elapsed_time(e1))
    assert lib.device_status() == 0, "a kernel wait gave up during warm-up"
    dominant = max(kern, key=lambda n: statistics.median(kern[n]))
    dom_idx = next(h for h in hooks if launched_kernel(w, h) == dominant)
    return kern, dominant, dom_idx, statistics.median(steps_ms)


def dominant_ms(kern, dominant, starts, stops, graphs, w, ms_step) -> float:
    """Mean time of the dominant kernel.  Host launches: the library's events
    around it in every timed step.  Graph replay: the hook records outside
    graphs, so the warm-up's events are used, except for a step of one launch,
    where the replayed step itself bounds the kernel's time from above (the
    warm-up events also hold the host's launch latency, which a graph hides)."""
    if not graphs:
        return statistics.fmean(a.elapsed_time(b) for a, b in zip(starts, stops))
    warm = statistics.fmean(kern[dominant])
    return min(warm, ms_step) if launches_per_step(w) == 1 else warm


def auto_steps(step_ms: float, seconds: float) -> int:
    """Timed steps that take about the given time at the warm-up's step time."""
    return max(5, min(2000, int(seconds * 1e3 / max(step_ms, 1e-3))))


def compare_variants(args, w):
    """Workloads run after the headline one for the same-kernel head-layout
    comparison (the same model with every head kept, GQA and MQA)."""
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    if args.no_compare:
        return []
    groups = {"large_dh128": ("large_dh128_mha", "large_dh128_gqa", "large_dh128_mqa"),
              "sqatm_block_sqa": ("sqatm_block_mha", "sqatm_block_gqa", "sqatm_block_mqa"),
              "sqatm_train_sqa": ("sqatm_train_mha", "sqatm_train_gqa", "sqatm_train_mqa"),
              "enc32k_8_4": ("enc32k_16_16", "enc32k_16_4", "enc32k_16_1", "enc32k_8_8", "enc32k_4_4")}
    return [WORKLOADS[n] for n in groups.get(w.name, ())]


def time_variant(args, lib, w, torch, world, rank, peaks, peak_kind):
    """Device time of the same kernels on another head layout: warm-up, then
    args.steps steps with the dominant kernel timed by the library hook."""
    from sparse_query_attention_sqa_b200.inputs import workload_inputs

    ev = lambda: torch.cuda.Event(enable_timing=True)
    q, k, v, dout = workload_inputs(w, seed=rank)
    first = alloc_set(w, q, k, v, dout, lib, torch)
    n_sets = max(2, math.ceil(2 * L2_BYTES / set_bytes(first)))
    sets = [first] + [alloc_set(w, q, k, v, dout, lib, torch) for _ in range(n_sets - 1)]
    del q, k, v, dout
    kern, dominant, dom_idx, warm_ms = warm_up(lib, w, sets, args.warmup, torch)
    graphs = graph_steps(lib, w, sets, torch, args)
    n_steps = (auto_steps(max_over_ranks(warm_ms, world, "cuda"), 8.0) if getattr(args, "steps_auto", False)
               else args.steps)
    if graphs:
        graphs.prepare(n_steps)
    starts = [ev() for _ in range(n_steps)]
    stops = [ev() for _ in range(n_steps)]
    t0, t1 = ev(), ev()
    torch.cuda.synchronize()
    t0.record()
    if graphs:
        graphs.run(n_steps)
    else:
        for i in range(n_steps):
            lib.set_timing_events(dom_idx, starts[i], stops[i])
            step(lib, w, sets[i % n_sets])
    t1.record()
    lib.set_timing_events(dom_idx)
    torch.cuda.synchronize()
    assert lib.device_status() == 0, "a kernel wait gave up while timing a comparison layout"
    ms_step = max_over_ranks(t0.elapsed_time(t1), world, "cuda") / n_steps
    dom_ms = dominant_ms(kern, dominant, starts, stops, graphs, w, ms_step)
    rl = roofline_for(w, dominant, dom_ms, peaks, peak_kind)
    rl.pop("traffic", None)
    out = {"workload": w.name, "H_q": w.Hq, "H_kv": w.Hkv, "steps": n_steps, "ms_per_step": ms_step,
           "value": job_tflops(w, world, ms_step), "unit": "TFLOP/s",
           "kernel_ms": {n: statistics.median(v) for n, v in kern.items()}, "roofline": rl}
    del sets
    torch.cuda.empty_cache()
    return out


def shard_inputs(w, world, rank):
    """This rank's part of one problem split by (batch entry, KV head): the
    workload of its block and the block of the problem's inputs (drawn whole
    with seed 0 on every rank, then sliced, so the blocks together are the
    problem)."""
    import dataclasses

    from sparse_query_attention_sqa_b200 import shard
    from sparse_query_attention_sqa_b200.inputs import workload_inputs

    if w.decode or w.block:
        raise SystemExit("--shard splits attention forward / backward workloads only")
    blk = shard.shard_block(w.B, w.Hkv, world, rank)
    g = w.Hq // w.Hkv
    part = dataclasses.replace(w, B=blk.b1 - blk.b0, Hq=g * (blk.k1 - blk.k0), Hkv=blk.k1 - blk.k0)
    q, k, v, dout = workload_inputs(w, seed=0)
    qh, kh = shard.q_heads(blk, g), shard.kv_heads(blk)
    return part, (shard.take(q, blk, qh), shard.take(k, blk, kh), shard.take(v, blk, kh),
                  shard.take(dout, blk, qh) if dout is not None else None)


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import sparse_query_attention_sqa_b200 as lib
    from sparse_query_attention_sqa_b200.inputs import workload_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    lib.load_library()

    w_job = w
    if args.shard and world > 1:
        # One problem over the ranks: this rank's (batch entry, KV head) block of it.
        w, (q, k, v, dout) = shard_inputs(w_job, world, rank)
    else:
        q, k, v, dout = workload_inputs(w, seed=rank)
    first = alloc_set(w, q, k, v, dout, lib, torch)
    n_sets = max(2, math.ceil(2 * L2_BYTES / set_bytes(first)))
    sets = [first] + [alloc_set(w, q, k, v, dout, lib, torch) for _ in range(n_sets - 1)]

    ev = lambda: torch.cuda.Event(enable_timing=True)
    kern, dominant, dom_idx, warm_ms = warm_up(lib, w, sets, args.warmup, torch)
    graphs = graph_steps(lib, w, sets, torch, args)
    if args.steps is None:  # every rank times the same number of steps
        args.steps = auto_steps(max_over_ranks(warm_ms, world, "cuda"), 20.0)
        args.steps_auto = True
    if graphs:
        graphs.prepare(args.steps)

    # Timed region: K steps, per-step events around the dominant kernel (graph
    # replays instead for launch-bound workloads; the dominant kernel's time is
    # then the warm-up's).
    starts = [ev() for _ in range(args.steps)]
    stops = [ev() for _ in range(args.steps)]
    t0, t1 = ev(), ev()
    clocks = ClockSampler(not args.no_clocks and rank == 0, local)
    time.sleep(0.2 if clocks.proc else 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    t0.record()
    if graphs:
        graphs.run(args.steps)
    else:
        for i in range(args.steps):
            lib.set_timing_events(dom_idx, starts[i], stops[i])
            step(lib, w, sets[i % n_sets])
    t1.record()
    lib.set_timing_events(dom_idx)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clk = clocks.stop()
    ms_total = max_over_ranks(t0.elapsed_time(t1), world, "cuda")
    assert lib.device_status() == 0, "a kernel wait gave up during the timed region"
    ms_step = ms_total / args.steps
    dom_ms = dominant_ms(kern, dominant, starts, stops, graphs, w, ms_step)
    sharded = w_job is not w
    value = counted_flops(w_job) / (ms_step * 1e-3) / 1e12 if sharded else job_tflops(w, world, ms_step)
    peaks, peak_kind = load_peaks()

    # End to end through the public API with host buffers: every step copies its
    # inputs in from pinned host memory, runs, and copies all of its outputs
    # back, all inside the timed region.  Consecutive steps rotate over up to
    # three streams, each with its own device buffers and host outputs, so one
    # step's copies overlap the others' kernels and copies (the link carries both
    # directions at once) -- the way a caller pipelines a stream of batches.
    n_pipe = min(3, n_sets)
    streams = [torch.cuda.Stream() for _ in range(n_pipe)]
    # (A decoding step's input is the new token's queries; its key/value cache
    # stays resident on the device, as in serving.)
    in_names = ("x", "dy") if w.block else (("q",) if w.decode else ("q", "k", "v", "dout"))
    host_in = {n: sets[0][n].cpu().pin_memory() for n in in_names if n in sets[0]}
    outs = ("y", "dx") if w.block else (("out", "lse", "dq", "dk", "dv") if w.backward else ("out", "lse"))
    host_out = [{n: torch.empty(sets[0][n].shape, dtype=sets[0][n].dtype, pin_memory=True) for n in outs}
                for _ in range(n_pipe)]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    e_steps = max(3, min(args.e2e_steps, args.steps))

    def e2e_step(i):
        k = i % n_pipe
        s = sets[k]
        with torch.cuda.stream(streams[k]):
            for n, t in host_in.items():
                s[n].copy_(t, non_blocking=True)
            step(lib, w, s)
            for n in outs:
                host_out[k][n].copy_(s[n], non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a, b = ev(), ev()
    a.record(streams[0])
    for st in streams[1:]:
        st.wait_event(a)
    for i in range(e_steps):
        e2e_step(i)
    for st in streams[1:]:
        streams[0].wait_stream(st)
    b.record(streams[0])
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e_steps, world, "cuda")
    if world > 1:
        dist.barrier()

    line = None
    if rank == 0:
        wj = w_job
        parallelism = (f"{world} ranks, each a (batch entry, KV head) block of one problem, no exchange" if sharded
                       else f"{world} independent replicas" if world > 1 else "single GPU")
        line = {
            "metric": f"{metric_name(wj)} {pass_name(wj)} TFLOP/s ({wj.note})",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Gaussian bf16 inputs)",
            "config": {"workload": wj.name, "B": wj.B, "N": wj.N, "H_q": wj.Hq, "H_kv": wj.Hkv, "dh": wj.dh,
                       "causal": wj.causal, "pass": pass_name(wj),
                       "parallelism": parallelism,
                       "l2": f"{n_sets} rotating buffer sets of {set_bytes(first) / 2**20:.0f} MiB "
                             f"(> L2 in total), no flush",
                       "launch": (f"CUDA-graph replay, {graphs.per} step(s) per graph" if graphs
                                  else "host launches"),
                       **({"d": w.d, "hidden": w.hidden, "layers": w.layers,
                           "weights": "random, one set shared by every block"} if w.block else {})},
            "tokens_per_s": (w_job.B * w_job.N if sharded else (w.B if w.decode else w.B * w.N) * world)
                            / (ms_step * 1e-3),
            "tensor_frac_of_bf16_peak": value / peaks["bf16_tflops"],
            "roofline": roofline_for(w, dominant, dom_ms, peaks, peak_kind),
            "kernel_ms": {n: statistics.median(v) for n, v in kern.items()},
            "e2e": {"value": (counted_flops(w_job) / (e2e_ms * 1e-3) / 1e12 if sharded
                              else job_tflops(w, world, e2e_ms)), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "streams": n_pipe,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": args.steps * launches_per_step(w),
            "clocks": clk,
            "wall_s_timed_region": wall,
            # the CUDA sources this run was built from (profiles/traffic.json entries are keyed to it)
            "source_sha256": kernel_source_sha256(),
        }
    # The same kernels on the MHA / GQA / MQA head layouts of the same model.
    variants = [] if sharded else compare_variants(args, w)
    if variants:
        sets.clear()
        first = host_in = host_out = None
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        comp = [time_variant(args, lib, v, torch, world, rank, peaks, peak_kind) for v in variants]
        if rank == 0:
            line["compare"] = comp
    # CPU baseline: rank 0 at N=1 only, after all GPU work.
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return None
    if not w.decode and (w.Hq // w.Hkv) * w.N * w.N * w.dh > 2 ** 34:  # one slice would take minutes: sample rows
        cb = cpu_baseline_rows(w, 60.0)
        return {"impl": "reference", "metric": f"{metric_name(w)} {pass_name(w)} TFLOP/s ({w.note})",
                "value": cb["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": 1, "warmup": 0,
                "ms_per_step": None, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "N": w.N, "H_q": w.Hq, "H_kv": w.Hkv, "dh": w.dh,
                           "causal": w.causal, "pass": pass_name(w)},
                "cpu_baseline": cb, "e2e": {"value": cb["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                                            "d2h_bytes_per_step": 0}}
    sub, data = oracle_subproblem(w)
    # Each step is the oracle's fwd(+bwd) on one batch entry's first KV group.
    # Cap the executed steps so the whole run stays within a few minutes.
    run_oracle_step(sub, data)
    t = time.perf_counter()
    run_oracle_step(sub, data)
    one = time.perf_counter() - t
    budget = 150.0
    warm = min(args.warmup, max(0, int(0.1 * budget / one)))
    requested = args.steps if args.steps is not None else 2000
    steps = max(1, min(requested, int(0.9 * budget / one)))
    for _ in range(warm):
        run_oracle_step(sub, data)
    t0 = time.perf_counter()
    for _ in range(steps):
        run_oracle_step(sub, data)
    el = time.perf_counter() - t0
    ms = el / steps * 1e3
    value = counted_flops(sub) / (ms * 1e-3) / 1e12
    sample = (f"fp64 oracle {pass_name(w)} on batch entry 0, KV head 0 and its {sub.Hq} "
              f"query heads (N={w.N}, dh={w.dh}); {steps} of the requested {requested} steps run")
    return {"impl": "reference", "metric": f"{metric_name(w)} {pass_name(w)} TFLOP/s ({w.note})",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "H_q": w.Hq, "H_kv": w.Hkv, "dh": w.dh,
                       "causal": w.causal, "pass": pass_name(w)},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": omp_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    w = WORKLOADS[args.workload]
    line = run_reference(args, w) if args.impl == "reference" else run_ours(args, w)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
