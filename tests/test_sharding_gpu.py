"""Tensor-parallel head sharding on one GPU: every shard is an ordinary decode.

"Grouped-Query Attention (GQA) and Multi-Query Attention (MQA): Mathematical
Foundations, ...", section 4 "Tensor Parallelism (TP) Head Partitioning": with
H_KV % N = 0 each rank runs GQA on its own KV heads and their query heads; with
N > H_KV the KV heads are duplicated and each rank runs MQA on one of them.
Here the N shards run one after another as independent calls on one GPU (no
shard waits on another) and their outputs, concatenated along the head axis,
must match the oracle and the unsharded call.

Multi-token step: the concatenated shards equal the unsharded call bit for
bit.  Its kernel has no split-KV: a query row's scores, weights and value
sums run over the same 128-key steps in the same order whatever other rows
share its tile, so neither the head count of a shard nor the tile shape
changes a single bit.

Decode step: the shards agree with the unsharded call within 1e-4, not bit for
bit.  The decode schedule cuts the whole batch's tiles into equal shares per
CTA, so where a unit's split-KV boundaries fall (and with them the rounding of
its partial sums and their merge) depends on the total tile count, which a
shard changes.  Both sides are independently within the oracle tolerance.
"""

import dataclasses

import pytest
import torch

import gqa_mqa_kv_b200 as gq
from gqa_mqa_kv_b200.sharding import tp_head_shard
from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs
from tests.helpers import assert_parity, to_device
from tests.test_parity_gpu import oracle_full, run_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,h_q,h_kv", [(2, 64, 8), (8, 64, 8), (8, 32, 4), (4, 32, 1), (4, 32, 2)])
def test_tp_shards_reassemble_the_full_step(cuda_device, world, h_q, h_kv):
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged"], B=3, H_Q=h_q, H_KV=h_kv, seq_len=900)
    inp = make_inputs(w)
    d = to_device(inp, cuda_device)
    parts = []
    for rank in range(world):
        qs, ks = tp_head_shard(h_q, h_kv, world, rank)
        q = d["q"][:, qs].contiguous()
        k = d["k"][:, :, ks].contiguous()
        v = d["v"][:, :, ks].contiguous()
        parts.append(gq.gqa_decode(q, k, v, d["seq_lens"], scale=w.softmax_scale))
    got = torch.cat(parts, dim=1).cpu()
    assert_parity(got, oracle_full(inp, w), f"TP {world} over {h_q}/{h_kv}")
    full = run_gpu(inp, w, cuda_device)
    assert (got - full).abs().max().item() < 1e-4  # split boundaries differ (module docstring)


@pytest.mark.parametrize("world,h_q,h_kv", [(2, 64, 8), (8, 32, 4), (4, 32, 2)])
def test_tp_prefill_shards_reassemble_the_full_step(cuda_device, world, h_q, h_kv):
    # The multi-token step shards the same way; every shard is an ordinary
    # gqa_prefill call on its query heads and their (possibly duplicated) KV heads.
    import numpy as np

    import oracle
    from gqa_mqa_kv_b200.workloads import PrefillWorkload, make_prefill_inputs

    w = PrefillWorkload("tp", 3, h_q, h_kv, 128, 1, 0, seed=32)
    n, L = np.array([150, 1, 70]), np.array([150, 260, 300])
    inp = make_prefill_inputs(w, pad_value=float("nan"), lengths=(n, L))
    d = to_device(inp, cuda_device)
    parts = []
    for rank in range(world):
        qs, ks = tp_head_shard(h_q, h_kv, world, rank)
        parts.append(gq.gqa_prefill(d["q"][:, qs].contiguous(), d["k"][:, :, ks].contiguous(),
                                    d["v"][:, :, ks].contiguous(), d["seq_lens"], d["cu_q"], max_q_len=d["max_q"]))
    got = torch.cat(parts, dim=1).cpu()
    ref = oracle.gqa_prefill(inp["q"], inp["k"], inp["v"], inp["seq_lens"], inp["cu_q"], w.softmax_scale)
    assert_parity(got, ref, f"TP prefill {world} over {h_q}/{h_kv}")
    full = gq.gqa_prefill(d["q"], d["k"], d["v"], d["seq_lens"], d["cu_q"], max_q_len=d["max_q"]).cpu()
    assert torch.equal(got.view(torch.int32), full.view(torch.int32)), "prefill shards differ from the whole call"
