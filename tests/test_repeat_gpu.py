"""Many back-to-back calls on one workspace (GPU).

Every decode call cuts units across CTAs and merges their partials inside the
split kernel with counters that alternate between two banks from call to call;
the multi-token kernel keeps only its status word there.  Hundreds of calls in
a row on one workspace, with no synchronisation between them, must give
bit-identical outputs and raise no status flag (a lost or doubled merge ticket
would leave a unit unmerged or merged from a stale partial, and a wait that
ran out would raise GQA_FLAG_TIMEOUT).
"""

import dataclasses

import pytest
import torch

import gqa_mqa_kv_b200 as gq
from gqa_mqa_kv_b200 import workloads as W
from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CALLS = 300


def _repeat(run, ws):
    first = run().clone()
    differ = sum(not torch.equal(run().view(torch.uint8), first.view(torch.uint8)) for _ in range(CALLS))
    assert differ == 0, f"{differ} of {CALLS} repeated calls changed the output"
    assert gq.read_status(ws) == 0


def _device(inp, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


@pytest.mark.parametrize("name,kernel,batch", [("llama2_70b_ragged", "auto", 12), ("llama3_8b", "auto", None),
                                               ("sweep_hkv1", "auto", 8), ("sweep_hkv2", "auto", 8),
                                               ("llama3_8b", "tcgen05", None)])
def test_decode_repeats_bitwise(cuda_device, name, kernel, batch):
    w = WORKLOADS[name] if batch is None else dataclasses.replace(WORKLOADS[name], B=batch)
    d = _device(make_inputs(w), cuda_device)
    ws = gq.make_workspace(gq.make_params(d["q"], d["k"], d["seq_lens"]), cuda_device).zero_()
    out = torch.empty(d["q"].shape, dtype=torch.float32, device=cuda_device)
    _repeat(lambda: gq.gqa_decode(d["q"], d["k"], d["v"], d["seq_lens"], scale=w.softmax_scale, out=out,
                                  workspace=ws, kernel=kernel), ws)


@pytest.mark.parametrize("name,batch", [("llama3_8b_fp8", None), ("llama2_70b_ragged_fp8", 12)])
def test_fp8_decode_repeats_bitwise(cuda_device, name, batch):
    w = WORKLOADS[name] if batch is None else dataclasses.replace(WORKLOADS[name], B=batch)
    d = _device(make_inputs(w), cuda_device)
    ws = gq.make_workspace(gq.make_params(d["q"], d["k"], d["seq_lens"]), cuda_device).zero_()
    out = torch.empty(d["q"].shape, dtype=torch.float32, device=cuda_device)
    _repeat(lambda: gq.gqa_decode_fp8kv(d["q"], d["k"], d["v"], d["k_scale"], d["v_scale"], d["seq_lens"],
                                        scale=w.softmax_scale, out=out, workspace=ws), ws)


def test_prefill_repeats_bitwise(cuda_device):
    w = W.PREFILL_WORKLOADS["prefill_ragged_paged"]
    inp = W.make_prefill_inputs(w)
    d = _device(inp, cuda_device)
    proxy = torch.empty((w.B, w.H_Q, w.D), dtype=torch.bfloat16, device="meta")
    ws = torch.zeros_like(gq.make_workspace(gq.make_params(proxy, d["k_paged"], d["seq_lens"], d["block_table"]),
                                            cuda_device))
    out = torch.empty((d["q"].shape[0], w.H_Q, w.D), dtype=torch.bfloat16, device=cuda_device)
    _repeat(lambda: gq.gqa_prefill(d["q"], d["k_paged"], d["v_paged"], d["seq_lens"], d["cu_q"],
                                   max_q_len=inp["max_q"], block_table=d["block_table"], out=out, workspace=ws), ws)
