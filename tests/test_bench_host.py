"""Host logic of bench.py that needs no GPU: the source hash that decides
whether a committed DRAM-traffic capture still describes the kernels."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_comments_are_removed_and_literals_kept():
    src = 'int a = 1; // note\n/* block\n */ const char* s = "x // y /* z */"; char c = \'"\'; int d;'
    out = bench.strip_c_comments(src)
    assert "note" not in out and "block" not in out
    assert '"x // y /* z */"' in out and "'\"'" in out and "int d;" in out


def test_comment_edits_keep_the_hash_and_code_edits_change_it():
    a = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    b = "int f(int x) {\n  return x + 1;  // increment\n}\n"
    c = "int f(int x) {\n  return x + 2;  // add one\n}\n"
    assert bench.strip_c_comments(a) == bench.strip_c_comments(b)
    assert bench.strip_c_comments(a) != bench.strip_c_comments(c)


def test_comment_and_layout_edits_keep_the_source_hash(tmp_path, monkeypatch):
    csrc = tmp_path / "sparse_query_attention_sqa_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_text("// one line\nint f(int x) { return x + 1; }\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_sha256()
    (csrc / "k.cuh").write_text("// a comment\n// of two lines\nint f(int x) {\n  return x + 1;\n}\n")
    assert bench.kernel_source_sha256() == h0
    (csrc / "k.cuh").write_text("int f(int x) { return x - 1; }\n")
    assert bench.kernel_source_sha256() != h0


def test_traffic_table_names_a_capture_command_per_entry():
    import json

    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    for e in table["entries"]:
        assert e["command"].startswith("ncu ") and "--clock-control none" in e["command"]
        assert e["dram_bytes_per_launch"] > 0 and len(e["source_sha256"]) == 64


def test_reference_arm_prints_one_complete_json_line():
    import json
    import subprocess

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "sqatm_layer_fwd", "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "sqatm_layer_fwd"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_roofline_reports_the_stated_algorithmic_work():
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0}
    ms = 0.5
    # decode: HBM-bound on the caches plus q, out and lse
    w = WORKLOADS["decode_sqatm"]
    rl = bench.roofline_for(w, "sqa_decode_split_kernel", ms, peaks, "measured")
    want = (2 * w.B * w.N * w.Hkv * w.dh * 2 + 2 * w.B * w.Hq * w.dh * 2 + 4 * w.B * w.Hq) / (ms * 1e-3) / 1e9
    assert rl["bound"] == "hbm" and rl["unit"] == "GB/s" and rl["peak"] == 6000.0
    assert abs(rl["achieved"] - want) < 1e-6 * want and abs(rl["frac"] - want / 6000.0) < 1e-12
    # dh 16: one exp2 per unmasked score element against the derived special-function peak
    w = WORKLOADS["sqatm_train_sqa"]
    rl = bench.roofline_for(w, "sqa_bwd_kernel", ms, peaks, "measured")
    causal_pairs = w.B * w.Hq * w.N * (w.N + 1) / 2
    assert rl["bound"] == "alu" and rl["unit"] == "Gexp2/s"
    assert abs(rl["achieved"] - causal_pairs / (ms * 1e-3) / 1e9) < 1e-6 * rl["achieved"]
    assert abs(rl["peak"] - 148 * 16 * 1965e6 / 1e9) < 1e-9
    for rl in (bench.roofline_for(WORKLOADS[n], k, ms, peaks, "measured")
               for n, k in (("decode_sqatm", "sqa_decode_split_kernel"), ("sqatm_train_sqa", "sqa_fwd_kernel"))):
        assert set(rl) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}


def test_launched_kernel_names_the_decoding_path_that_runs():
    # the same selection rule as the library: register-resident (g <= 4, H_kv a
    # power of two within one CTA step), tensor cores (5 <= g <= 16), else shared memory
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    assert bench.launched_kernel(WORKLOADS["decode_sqatm"], 2) == "sqa_decode_split_kernel<16,2>"
    assert bench.launched_kernel(WORKLOADS["decode_dh128"], 2) == "sqa_decode_split_kernel<128,2>"
    assert bench.launched_kernel(WORKLOADS["decode_mqa"], 2) == "sqa_decode_mma_kernel<16>"
    assert bench.launched_kernel(WORKLOADS["large_dh128"], 1) == "sqa_bwd_kernel<128,false>+sqa_bwd_q_kernel<128>"
    assert bench.launched_kernel(WORKLOADS["large_dh128_mqa"], 1) == "sqa_bwd_kernel<128,true>+sqa_bwd_q_kernel<128>"
    assert bench.launched_kernel(WORKLOADS["sqatm_train_sqa"], 1) == "sqa_bwd_tf32_kernel<16>"


def test_block_stack_counts_attention_and_matrix_products():
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    w = WORKLOADS["sqatm_block_sqa"]
    attn = 4.0 * 32 * 8 * 1024 * 1024 * 16 / 2 * 3.5
    params = 256 * (8 + 8) * 16 + 8 * 16 * 256 + 3 * 256 * 768
    assert bench.block_gemm_params(w) == params
    assert bench.counted_flops(w) == 8 * (attn + 2.0 * 32 * 1024 * params * 3)
    assert bench.launches_per_step(w) == 8 * 27
    assert bench.launches_per_step(WORKLOADS["large_dh128"]) == 4
    assert bench.pass_name(w) == "8-block fwd+bwd"
    # the MHA stack does the same matrix products as SQAT-m plus wider attention ones
    m = WORKLOADS["sqatm_block_mha"]
    assert bench.block_gemm_params(m) - params == 256 * (16 + 32 - 16) * 16 + 8 * 16 * 256


def test_default_step_count_follows_the_warm_up_time():
    """Without --steps the timed region lasts about the given time: 20 s of
    68.5 ms steps is 291 steps; very short steps stop at 2000, very long ones
    keep at least 5."""
    import bench

    assert bench.auto_steps(68.5, 20.0) == 291
    assert bench.auto_steps(0.01, 20.0) == 2000
    assert bench.auto_steps(10_000.0, 20.0) == 5


def test_graph_replayed_single_launch_step_bounds_the_kernel_time():
    """With CUDA-graph replay the hook's warm-up events include the host's
    launch latency; for a one-launch step the replayed step time is the
    tighter bound, for longer steps the warm-up's kernel time stands."""
    import bench
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    kern = {"k": [0.018, 0.018]}
    assert bench.dominant_ms(kern, "k", [], [], True, WORKLOADS["sqatm_layer_fwd"], 0.0135) == 0.0135
    assert bench.dominant_ms(kern, "k", [], [], True, WORKLOADS["sqatm_block_sqa"], 7.17) == 0.018


def test_graph_steps_replay_exactly_k_steps(monkeypatch):
    """Graphs of several one-launch steps: run(k) replays exactly k steps, the
    last k % per_graph of them from a graph captured before timing; each graph
    walks consecutive buffer sets."""
    import contextlib
    import types

    import bench

    log = {"captured": [], "replayed": 0, "current": None}

    class FakeGraph:
        def __init__(self):
            self.steps = []

        def replay(self):
            log["replayed"] += len(self.steps)

    @contextlib.contextmanager
    def graph(g, capture_error_mode=None):
        log["current"] = g
        yield
        log["current"] = None

    cuda = types.SimpleNamespace(CUDAGraph=FakeGraph, graph=graph, synchronize=lambda: None)
    fake_torch = types.SimpleNamespace(cuda=cuda)
    lib = types.SimpleNamespace(device_status=lambda: 0)
    monkeypatch.setattr(bench, "step", lambda lib_, w, s: log["current"].steps.append(s))
    sets = list(range(37))
    gs = bench.GraphSteps(lib, None, sets, fake_torch, 16)
    assert [g.steps for g in gs.graphs][:2] == [list(range(16)), list(range(16, 32))]
    assert gs.graphs[2].steps == [32, 33, 34, 35, 36] + list(range(11))
    for k in (1, 16, 2000, 2001, 37 * 16 + 5):
        gs.prepare(k)
        log["replayed"] = 0
        gs.run(k)
        assert log["replayed"] == k


def test_shard_inputs_split_one_problem_by_kv_head():
    """--shard: the two ranks' parts of the SQAT-m layer forward (B=1, 8/4)
    are query heads 0-3 with KV heads 0-1 and query heads 4-7 with KV heads
    2-3 of the same inputs; together they are the whole problem."""
    import torch

    import bench
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS, workload_inputs

    w = WORKLOADS["sqatm_layer_fwd"]
    q, k, v, _ = workload_inputs(w, seed=0)
    parts = [bench.shard_inputs(w, 2, r) for r in range(2)]
    assert [(p.B, p.Hq, p.Hkv) for p, _ in parts] == [(1, 4, 2), (1, 4, 2)]
    assert torch.equal(torch.cat([t[0] for _, t in parts], dim=2), q)
    assert torch.equal(torch.cat([t[1] for _, t in parts], dim=2), k)
    assert torch.equal(torch.cat([t[2] for _, t in parts], dim=2), v)
    assert sum(bench.counted_flops(p) for p, _ in parts) == bench.counted_flops(w)
