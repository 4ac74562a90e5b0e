"""Failure detection on the GPU without a fault: the bounded wait runs out.

gqa_wait_selftest makes the pipeline-barrier wait every kernel uses wait on an
mbarrier that nothing arrives on.  The wait must give up at its limit, raise
GQA_FLAG_TIMEOUT and return; an abort raised by another warp must end it
early; and the context must stay usable for a normal decode afterwards.
"""

import dataclasses

import pytest
import torch

import gqa_mqa_kv_b200 as gq
from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs
from tests.helpers import assert_parity
from tests.test_parity_gpu import oracle_full, run_gpu

pytestmark = pytest.mark.gpu


def test_wait_gives_up_at_its_limit(cuda_device):
    limit = 2_000_000  # 2 ms
    flags, elapsed = gq.wait_selftest(limit, device=cuda_device)
    assert flags & gq.FLAG_TIMEOUT
    assert limit <= elapsed < limit + 200_000_000


def test_abort_from_another_warp_ends_the_wait_early(cuda_device):
    limit = 400_000_000  # 0.4 s; the abort comes after a quarter of it
    flags, elapsed = gq.wait_selftest(limit, abort_early=True, device=cuda_device)
    assert flags & gq.FLAG_TIMEOUT
    assert limit // 4 <= elapsed < limit // 2


def test_context_stays_usable_after_timeouts(cuda_device):
    gq.wait_selftest(1_000_000, device=cuda_device)
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged"], B=3, seq_len=700)
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device), oracle_full(inp, w), "decode after a timeout")
    assert torch.cuda.is_available()
