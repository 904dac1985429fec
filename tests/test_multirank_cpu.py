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


def _shard_main(rank, world, port, out_dir):
    """Each rank computes its (batch entry, KV head) block of one problem with
    the oracle; the blocks travel to rank 0 over gloo."""
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import oracle
    from sparse_query_attention_sqa_b200 import shard
    from sparse_query_attention_sqa_b200.inputs import make_inputs

    got = {}
    for B, N, Hq, Hkv, dh in ((1, 40, 8, 4, 16), (2, 33, 6, 1, 16)):
        g = Hq // Hkv
        q, k, v, dout = make_inputs(B, N, Hq, Hkv, dh, seed=9, with_dout=True)
        blk = shard.shard_block(B, Hkv, world, rank)
        qs, ks, vs = (shard.take(t, blk, h) for t, h in ((q, shard.q_heads(blk, g)), (k, shard.kv_heads(blk)),
                                                        (v, shard.kv_heads(blk))))
        dos = shard.take(dout, blk, shard.q_heads(blk, g))
        out, lse = oracle.sqa_fwd(qs, ks, vs, True)
        dq, dk, dv = oracle.sqa_bwd(qs, ks, vs, dos, True)
        parts = [torch.from_numpy(a).contiguous() for a in (out, lse, dq, dk, dv)]
        gathered = []
        for t in parts:
            bufs = [torch.empty(0)] * world
            dist.all_gather_object(bufs, t)
            gathered.append(bufs)
        got[(B, N, Hq, Hkv, dh)] = gathered
    if rank == 0:
        torch.save(got, os.path.join(out_dir, "shard.pt"))
    dist.barrier()
    dist.destroy_process_group()


def test_ranks_computing_blocks_of_one_problem_reassemble_it(tmp_path):
    """Two gloo ranks each take their (batch entry, KV head) block of one
    problem (KV heads 0-1 and 2-3 of B=1; batch entries 0 and 1 of an MQA
    problem), compute it with the oracle and send it to rank 0: put back in
    place, the blocks equal the whole problem computed at once, forward and
    backward, with no exchange between the blocks."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import oracle
    from sparse_query_attention_sqa_b200 import shard
    from sparse_query_attention_sqa_b200.inputs import make_inputs

    mp.start_processes(_shard_main, args=(2, _free_port(), str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    got = torch.load(tmp_path / "shard.pt")
    for (B, N, Hq, Hkv, dh), gathered in got.items():
        g = Hq // Hkv
        q, k, v, dout = make_inputs(B, N, Hq, Hkv, dh, seed=9, with_dout=True)
        ref_out, ref_lse = oracle.sqa_fwd(q, k, v, True)
        ref = (ref_out, ref_lse) + tuple(oracle.sqa_bwd(q, k, v, dout, True))
        for which, (whole, blocks) in enumerate(zip(ref, gathered)):
            full = np.full_like(whole, np.nan)
            for r in range(2):
                blk = shard.shard_block(B, Hkv, 2, r)
                if which == 1:  # lse [B, H_q, N]
                    full[blk.b0:blk.b1, shard.q_heads(blk, g)] = blocks[r].numpy()
                else:
                    heads = shard.kv_heads(blk) if which >= 3 else shard.q_heads(blk, g)
                    full[blk.b0:blk.b1, :, heads] = blocks[r].numpy()
            assert np.array_equal(full, whole), (B, N, Hq, Hkv, dh, which)


def test_shard_block_rules():
    sys.path.insert(0, ROOT)
    from sparse_query_attention_sqa_b200.shard import Block, shard_block

    assert [shard_block(1, 4, 2, r) for r in range(2)] == [Block(0, 1, 0, 2), Block(0, 1, 2, 4)]
    assert [shard_block(2, 4, 4, r) for r in range(4)] == [Block(0, 1, 0, 2), Block(0, 1, 2, 4), Block(1, 2, 0, 2),
                                                           Block(1, 2, 2, 4)]
    assert shard_block(8, 4, 2, 1) == Block(4, 8, 0, 4)
    assert shard_block(2, 1, 2, 1) == Block(1, 2, 0, 1)
    for bad in ((1, 4, 3, 0), (3, 2, 2, 0), (1, 6, 4, 0)):
        with pytest.raises(ValueError):
            shard_block(*bad)


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
