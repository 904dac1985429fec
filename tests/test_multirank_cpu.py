"""The multi-GPU host logic of bench.py, run as two gloo ranks on the CPU.

Under torchrun every rank runs an independent replica of the workload (the
path shards into independent (batch, KV-head group) problems, so there is no
collective on the data path).  What the ranks share is host logic: each rank
draws its own inputs, the step time is the maximum over ranks, and the job's
throughput counts the work of every rank.  These tests run that logic with two
processes over gloo.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS, make_decode_inputs, workload_inputs

    w = WORKLOADS["sqatm_layer_fwd"]
    # Step times that differ by rank: every rank must see the slowest one.
    ms = bench.max_over_ranks(1.0 + 0.25 * rank, world, "cpu")
    q, _, _, _ = workload_inputs(w, seed=rank)
    wd = WORKLOADS["decode_sqatm"]
    qd = make_decode_inputs(2, 64, wd.Hq, wd.Hkv, wd.dh, seed=rank)[0]
    torch.save({"ms": ms, "q": q, "qd": qd, "value": bench.job_tflops(w, world, ms),
                "value_decode": bench.job_tflops(wd, world, ms)}, os.path.join(out_dir, f"r{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    out = tmp_path_factory.mktemp("ranks")
    mp.start_processes(_rank_main, args=(2, _free_port(), str(out)), nprocs=2, start_method="spawn", join=True)
    return [torch.load(os.path.join(out, f"r{r}.pt")) for r in range(2)]


def test_step_time_is_the_maximum_over_ranks(two_ranks):
    assert [r["ms"] for r in two_ranks] == [1.25, 1.25]


def test_job_throughput_counts_every_rank(two_ranks):
    sys.path.insert(0, ROOT)
    import bench
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    w = WORKLOADS["sqatm_layer_fwd"]
    one = bench.job_tflops(w, 1, 1.25)
    assert two_ranks[0]["value"] == pytest.approx(2 * one)
    assert two_ranks[1]["value"] == pytest.approx(2 * one)


def test_ranks_draw_independent_inputs(two_ranks):
    for key in ("q", "qd"):
        a, b = two_ranks[0][key], two_ranks[1][key]
        assert a.shape == b.shape and a.dtype == torch.bfloat16
        assert not torch.equal(a, b)


def test_decoding_job_throughput_counts_every_rank(two_ranks):
    sys.path.insert(0, ROOT)
    import bench
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    w = WORKLOADS["decode_sqatm"]
    # one query row per (sequence, head) against the whole cache, on each rank
    per_rank = 4.0 * w.B * w.Hq * w.N * w.dh / 1.25e-3 / 1e12
    assert two_ranks[0]["value_decode"] == pytest.approx(2 * per_rank)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from sparse_query_attention_sqa_b200.inputs import WORKLOADS

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.run_reference(None, WORKLOADS["decode_sqatm"]) is None


def test_single_rank_reduction_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
