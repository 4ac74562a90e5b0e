"""Multi-rank host logic on CPU with world_size 2 gloo process groups.

Covers the benchmark's distributed plumbing (rank environment, max-over-ranks
timing, rank-0-only reference arm) and the partitioning helpers: batch shards
and tensor-parallel head shards, each checked by running the fp64 oracle on
every rank's shard and comparing the gathered result with the unsharded one.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, fn_name, out_q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        import bench  # noqa: F401  (imports must work on a CPU-only host)

        g = globals()[fn_name]
        res = g(rank, world)
        out_q.put((rank, "ok", res))
    except Exception as e:  # report to the parent instead of hanging it
        out_q.put((rank, "error", repr(e)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def run_ranks(fn_name, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fn_name, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, status, res = q.get(timeout=180)
        assert status == "ok", res
        results[rank] = res
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return results


def rank_timing(rank, world):
    import bench

    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    d = bench.init_dist(w, "gloo")
    t = bench.max_over_ranks(1.5 + rank, d, torch.device("cpu"))
    d.barrier()
    return t


def rank_batch_shards(rank, world):
    import oracle
    from gqa_mqa_kv_b200.sharding import batch_shard
    from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs
    import dataclasses

    dist.init_process_group("gloo")
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged"], B=5, seq_len=300)
    inp = make_inputs(w)
    sl = batch_shard(w.B, world, rank)
    mine = oracle.gqa_decode(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["seq_lens"][sl], w.softmax_scale)
    parts = [None] * world
    dist.all_gather_object(parts, (sl.start, mine))
    full = oracle.gqa_decode(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale)
    import numpy as np

    got = np.concatenate([p[1] for p in sorted(parts, key=lambda x: x[0])])
    return bool(np.array_equal(got, full))


def rank_tp_shards(rank, world):
    import numpy as np

    import oracle
    from gqa_mqa_kv_b200.sharding import tp_head_shard
    from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs
    import dataclasses

    dist.init_process_group("gloo")
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged"], B=3, seq_len=200)
    inp = make_inputs(w)
    qs, ks = tp_head_shard(w.H_Q, w.H_KV, world, rank)
    mine = oracle.gqa_decode(inp["q"][:, qs].contiguous(), inp["k"][:, :, ks].contiguous(),
                             inp["v"][:, :, ks].contiguous(), inp["seq_lens"], w.softmax_scale)
    parts = [None] * world
    dist.all_gather_object(parts, (qs.start, mine))
    got = np.concatenate([p[1] for p in sorted(parts, key=lambda x: x[0])], axis=1)
    full = oracle.gqa_decode(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale)
    return bool(np.array_equal(got, full))


def rank_tp_dup_shards(rank, world):
    import dataclasses

    import numpy as np

    import oracle
    from gqa_mqa_kv_b200.sharding import tp_head_shard
    from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs

    dist.init_process_group("gloo")
    # 4 ranks over 2 KV heads: each KV head is held by two ranks
    w = dataclasses.replace(WORKLOADS["tiny"], B=2, H_Q=8, H_KV=2, seq_len=96)
    inp = make_inputs(w)
    qs, ks = tp_head_shard(w.H_Q, w.H_KV, world, rank)
    mine = oracle.gqa_decode(inp["q"][:, qs].contiguous(), inp["k"][:, :, ks].contiguous(),
                             inp["v"][:, :, ks].contiguous(), inp["seq_lens"], w.softmax_scale)
    parts = [None] * world
    dist.all_gather_object(parts, (qs.start, mine))
    got = np.concatenate([m for _, m in sorted(parts, key=lambda x: x[0])], axis=1)
    full = oracle.gqa_decode(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale)
    return bool(np.array_equal(got, full))


def rank_tp_prefill_shards(rank, world):
    # The multi-token step shards by heads the same way: each rank runs the
    # causal step on its query heads and their (possibly duplicated) KV heads.
    import numpy as np

    import oracle
    from gqa_mqa_kv_b200.sharding import tp_head_shard
    from gqa_mqa_kv_b200.workloads import PrefillWorkload, make_prefill_inputs

    dist.init_process_group("gloo")
    w = PrefillWorkload("tp", 3, 8, 2, 16, 1, 0, seed=31)
    n, L = np.array([5, 1, 9]), np.array([12, 7, 9])
    inp = make_prefill_inputs(w, lengths=(n, L))
    qs, ks = tp_head_shard(w.H_Q, w.H_KV, world, rank)
    mine = oracle.gqa_prefill(inp["q"][:, qs].contiguous(), inp["k"][:, :, ks].contiguous(),
                              inp["v"][:, :, ks].contiguous(), inp["seq_lens"], inp["cu_q"], w.softmax_scale)
    parts = [None] * world
    dist.all_gather_object(parts, (qs.start, mine))
    got = np.concatenate([m for _, m in sorted(parts, key=lambda x: x[0])], axis=1)
    full = oracle.gqa_prefill(inp["q"], inp["k"], inp["v"], inp["seq_lens"], inp["cu_q"], w.softmax_scale)
    return bool(np.array_equal(got, full))


def rank_reference_arm(rank, world):
    import bench

    if rank != 0:
        return bench.run_reference(bench.parse_args(["--impl", "reference", "--gpus", str(world)]))
    return 0  # rank 0 would run the oracle; only the non-zero ranks' early exit is checked here


def test_max_over_ranks_with_gloo():
    res = run_ranks("rank_timing")
    assert res == {0: 2.5, 1: 2.5}


def test_batch_shards_reassemble_the_full_step():
    assert run_ranks("rank_batch_shards") == {0: True, 1: True}


def test_tensor_parallel_head_shards_reassemble_the_full_step():
    assert run_ranks("rank_tp_shards") == {0: True, 1: True}


def test_reference_arm_runs_on_rank_zero_only():
    assert run_ranks("rank_reference_arm") == {0: 0, 1: 0}


def rank_reference_arm_prefill(rank, world):
    import bench

    if rank != 0:
        return bench.main(["--impl", "reference", "--gpus", str(world), "--workload", "prefill_llama3_8b"])
    return 0  # only the non-zero ranks' early exit is checked here


def test_prefill_reference_arm_runs_on_rank_zero_only():
    assert run_ranks("rank_reference_arm_prefill") == {0: 0, 1: 0}


def test_shard_helpers():
    from gqa_mqa_kv_b200.sharding import batch_shard, tp_head_shard

    assert [batch_shard(7, 3, r) for r in range(3)] == [slice(0, 2), slice(2, 4), slice(4, 7)]
    assert tp_head_shard(64, 8, 8, 3) == (slice(24, 32), slice(3, 4))
    # TP > H_KV duplicates KV heads: 8 ranks over 4 KV heads, two ranks per head
    assert [tp_head_shard(32, 4, 8, r) for r in (0, 1, 2, 7)] == [
        (slice(0, 4), slice(0, 1)), (slice(4, 8), slice(0, 1)), (slice(8, 12), slice(1, 2)),
        (slice(28, 32), slice(3, 4))]
    with pytest.raises(ValueError):
        tp_head_shard(32, 4, 3, 0)  # neither divides the other
    with pytest.raises(ValueError):
        tp_head_shard(24, 8, 16, 0)  # H_Q not a multiple of the TP size


def test_duplicated_kv_shards_keep_each_query_head_on_its_own_group():
    from gqa_mqa_kv_b200.sharding import tp_head_shard

    for H_Q, H_KV, world in [(32, 4, 8), (64, 8, 16), (32, 1, 4), (64, 2, 32)]:
        R = H_Q // H_KV
        for rank in range(world):
            qs, ks = tp_head_shard(H_Q, H_KV, world, rank)
            assert ks.stop - ks.start == 1
            assert all(h // R == ks.start for h in range(qs.start, qs.stop))


def test_tensor_parallel_with_duplicated_kv_reassembles_the_full_step():
    assert run_ranks("rank_tp_dup_shards", world=4) == {0: True, 1: True, 2: True, 3: True}


def test_tensor_parallel_prefill_shards_reassemble_the_full_step():
    assert run_ranks("rank_tp_prefill_shards") == {0: True, 1: True}
    # four ranks over two KV heads: duplicated KV, one group slice per rank
    assert run_ranks("rank_tp_prefill_shards", world=4) == {0: True, 1: True, 2: True, 3: True}
